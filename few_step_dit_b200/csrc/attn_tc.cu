// Joint attention on the sm_100a tensor cores (bf16 operands, fp32 softmax).
//
// One CTA per (128-query tile, head); 192 threads:
//   warp 0  lane 0: TMA producer.  Q, K and V tiles are 128 x 128 boxes cut
//           straight out of the packed qkv buffer [n, 3A] (two 64-column
//           boxes each, 128-byte swizzle); K and V go through a 2-stage ring.
//   warp 1  allocates TMEM; lane 0 issues tcgen05.mma:
//           S[j%2] = Q K_j^T  (TMEM, fp32, double-buffered 2 x 128 columns),
//           O     += P_j V_j  (TMEM, fp32, 128 columns; V is an MN-major operand).
//   warps 2-5: softmax, one thread per query row (TMEM lane).  Each thread
//           reads its S row, keeps a running max m and sum l in the log2
//           domain, writes P = exp2(s*scale - m) as bf16 into shared memory
//           (the K-major 128B-swizzled layout the MMA reads), and rescales its
//           O row in TMEM only when its max grew by more than 8 (P stays
//           below 2^8, exact in fp32 accumulation).  At the end O / l is
//           stored as bf16.
// Keys past n are masked (the TMA zero-fills rows past n).
#include "tc_ptx.cuh"

namespace fsdit {
namespace attn {

constexpr int BQ = 128, BKV = 128, D = 128;
constexpr int TILE_BYTES = 128 * 128 * 2;  // 32 KB: two 64-column swizzled boxes
constexpr int HALF_BYTES = TILE_BYTES / 2;
constexpr int THREADS = 192;
constexpr int OFF_Q = 0;
constexpr int OFF_K0 = TILE_BYTES;         // K stage s at OFF_K0 + s * 2 * TILE_BYTES
constexpr int OFF_P = 5 * TILE_BYTES;
constexpr int OFF_BAR = 6 * TILE_BYTES;
// barriers: q_full, k_full[2], v_full[2], k_empty[2], v_empty[2], s_full[2], s_free[2], p_full, o_done
enum { B_QFULL = 0, B_KFULL = 1, B_VFULL = 3, B_KEMPTY = 5, B_VEMPTY = 7, B_SFULL = 9, B_SFREE = 11,
       B_PFULL = 13, B_ODONE = 14, NUM_BARS = 15 };
constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
constexpr uint32_t TMEM_COLS = 512;        // S0 [0,128), S1 [128,256), O [256,384)
constexpr uint32_t T_O = 256;
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
  const int q0 = blockIdx.x * BQ;
  const int n = args.n;
  const int nkv = (n + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
      mbar_init(bar(B_SFULL + s), 1);
      mbar_init(bar(B_SFREE + s), 128);
    }
    mbar_init(bar(B_PFULL), 128);
    mbar_init(bar(B_ODONE), 1);
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
      mbar_expect_tx(bar(B_QFULL), TILE_BYTES);
      tma_load_2d(base + OFF_Q, &tm, cq, q0, bar(B_QFULL));
      tma_load_2d(base + OFF_Q + HALF_BYTES, &tm, cq + 64, q0, bar(B_QFULL));
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        const uint32_t sk = base + OFF_K0 + st * 2 * TILE_BYTES, sv = sk + TILE_BYTES;
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
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        if (!mbar_wait(bar(B_KFULL + st), ph, abort_flag)) return false;
        if (!mbar_wait(bar(B_SFREE + st), ph ^ 1u, abort_flag)) return false;
        tc_fence_after();
        const uint32_t sk = base + OFF_K0 + st * 2 * TILE_BYTES;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (uint32_t)((k >> 2) * HALF_BYTES + (k & 3) * 32);
          mma_bf16_ss(tmem + (uint32_t)(st * BKV), sw128_desc(base + OFF_Q + off, 16, 1024),
                      sw128_desc(sk + off, 16, 1024), IDESC_S, k > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_KEMPTY + st));
        tc_commit(bar(B_SFULL + st));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < nkv && ok; ++j) {
        if (j + 1 < nkv && !issue_s(j + 1)) { ok = false; break; }
        const int st = j & 1;
        const uint32_t ph = (uint32_t)(j >> 1) & 1u;
        if (!mbar_wait(bar(B_PFULL), (uint32_t)j & 1u, abort_flag)) { ok = false; break; }
        if (!mbar_wait(bar(B_VFULL + st), ph, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sv = base + OFF_K0 + st * 2 * TILE_BYTES + TILE_BYTES;
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k) {
          const uint32_t pa = base + OFF_P + (uint32_t)((k >> 2) * HALF_BYTES + (k & 3) * 32);
          // V rows k*16 .. k*16+15: 2 groups of 8 rows of 128 B
          mma_bf16_ss(tmem + T_O, sw128_desc(pa, 16, 1024), sw128_desc(sv + (uint32_t)(k * 2048), HALF_BYTES, 1024),
                      IDESC_PV, (j > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(bar(B_VEMPTY + st));
        tc_commit(bar(B_ODONE));
      }
    }
  } else {
    // softmax warps: thread <-> query row r of the tile (TMEM lane r)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const float sl2 = args.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait(bar(B_SFULL + sb), (uint32_t)(j >> 1) & 1u, abort_flag) ? 1 : 0;
      w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
      if (!w_ok) { ok = false; break; }
      tc_fence_after();
      float s[BKV];
#pragma unroll
      for (int c = 0; c < BKV / 32; ++c) tmem_ld32(tmem + lane_addr + (uint32_t)(sb * BKV + c * 32), s + c * 32);
      tc_fence_before();
      mbar_arrive(bar(B_SFREE + sb));
      const int valid = n - j * BKV;  // keys past n are masked
      if (valid < BKV) {
#pragma unroll
        for (int c = 0; c < BKV; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < BKV; ++c) mx = fmaxf(mx, s[c]);
      const float m_cand = mx * sl2;
      // keep the old max unless it grew by more than the threshold
      const bool grow = m_cand > m + RESCALE_THRESHOLD;
      const float m_new = grow ? m_cand : m;
      const float corr = grow ? ex2(m - m_new) : 1.0f;
      float sum = 0.f;
      uint32_t pk[BKV / 2];
#pragma unroll
      for (int c = 0; c < BKV; c += 2) {
        const float p0 = ex2(fmaf(s[c], sl2, -m_new));
        const float p1 = ex2(fmaf(s[c + 1], sl2, -m_new));
        sum += p0 + p1;
        pk[c >> 1] = pack_bf16(p0, p1);
      }
      l = l * corr + sum;
      m = m_new;
      if (j > 0) {
        // P buffer and O are in use by PV_{j-1} until it completes
        if (lane == 0) w_ok = mbar_wait(bar(B_ODONE), (uint32_t)(j - 1) & 1u, abort_flag) ? 1 : 0;
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            const uint32_t ta = tmem + lane_addr + T_O + (uint32_t)(c * 32);
            tmem_ld32(ta, o);
            uint32_t u[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(o[i] * corr);
            tmem_st32(ta, u);
          }
        }
      }
      // P row r -> swizzled K-major tile: 16-byte chunk g holds keys 8g..8g+7
      uint8_t* prow = base_ptr + OFF_P + r * 128;
#pragma unroll
      for (int g = 0; g < BKV / 8; ++g) {
        const int half = g >> 3, ch = g & 7;
        uint4 v = make_uint4(pk[4 * g], pk[4 * g + 1], pk[4 * g + 2], pk[4 * g + 3]);
        *reinterpret_cast<uint4*>(prow + half * HALF_BYTES + ((ch ^ (r & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL));
    }
    if (ok && nkv > 0) {
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait(bar(B_ODONE), (uint32_t)(nkv - 1) & 1u, abort_flag) ? 1 : 0;
      w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
      if (w_ok) {
        tc_fence_after();
        const int row = q0 + r;
        const float inv = 1.0f / l;
        bf16* orow = args.out + (size_t)row * args.attn + head * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tmem + lane_addr + T_O + (uint32_t)(c * 32), o);
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
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(tc_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
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
  dim3 grid((n + BQ - 1) / BQ, heads);
  tc_attention_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tm, a);
  return cuda_check(cudaGetLastError(), "tc_attention_kernel");
}

}  // namespace fsdit
