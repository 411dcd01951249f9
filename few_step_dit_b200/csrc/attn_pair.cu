// Joint attention on the sm_100a tensor cores, CTA-pair form for long
// sequences (bf16 operands, fp32 softmax; same result as tc_attention_kernel).
//
// A cluster of two CTAs on neighbouring SMs takes 256 queries of one head;
// CTA rank r holds rows r*128 .. r*128+127.  Every MMA is
// tcgen05.mma.cta_group::2 (M = 256) issued by one thread of rank 0, and both
// take their A operand from tensor memory, so each SM reads only its half of
// B from shared memory (64 bytes per cycle at the tensor pipe's rate):
//   S(j)  = Q K_j^T   A = Q in TMEM (loaded once per CTA); N = 128 keys:
//                     rank r stages keys r*64 .. r*64+63 of block j (K-major);
//   O    += P(j) V_j  A = P(j) in TMEM, written over S(j) as bf16; N = 128
//                     head columns: rank r stages columns r*64 .. r*64+63 of
//                     V_j for all 128 keys (MN-major).
// Each CTA's TMEM: S buffers 0 and 1 (128 columns each), O (128), Q (64).
// S is double-buffered: while the softmax works on S(j), the tensor pipe runs
// PV(j-1) and S(j+1), so no softmax waits for a matrix product of its own
// tile and the pipe never waits for a softmax it does not need.  The pair
// halves every CTA's share of the key/value stream, and the shared memory,
// free of Q and P, holds deep K and V rings (the copies take several
// thousand cycles to land).
//
// Threads (192 per CTA): warp 0 lane 0 loads K and V with TMA (each CTA its
// own halves; completion counted on rank 0's barriers); warp 1 allocates
// TMEM and, on rank 0, lane 0 issues the MMAs; warps 2-5 (one per SM
// sub-partition, each owning its TMEM lane quarter) load Q into TMEM, then
// run the softmax, one thread per query row: running max and sum in the
// log2 domain, O rescaled only when a row max grows by more than 8.  Every
// wait is bounded (see tc_ptx.cuh).
#include "tc_ptx.cuh"

namespace fsdit {
namespace attn2 {

constexpr int BQ = 128, BKV = 128, D = 128;
constexpr int KH_BYTES = 64 * 128 * 2;  // this CTA's 64 keys x 128 columns: two 64-column boxes
constexpr int KH_HALF = KH_BYTES / 2;
constexpr int VH_BYTES = 128 * 64 * 2;  // 128 keys x this CTA's 64 columns: one box
constexpr int NS = 6;                   // K and V ring stages
constexpr int THREADS = 192;
constexpr int SOFTMAX_WARPS = 4;
constexpr int OFF_K = 0;                      // K stage s at OFF_K + s * KH_BYTES
constexpr int OFF_V = NS * KH_BYTES;          // V stage s at OFF_V + s * VH_BYTES
constexpr int OFF_BAR = OFF_V + NS * VH_BYTES;
enum {
  B_KFULL = 0,                // rank 0: both CTAs' K halves landed
  B_VFULL = B_KFULL + NS,     // rank 0: both CTAs' V halves landed
  B_KEMPTY = B_VFULL + NS,    // both CTAs: the S MMA reading the stage is done
  B_VEMPTY = B_KEMPTY + NS,   // both CTAs: the PV MMA reading the stage is done
  B_QREADY = B_VEMPTY + NS,   // rank 0: both CTAs' Q rows are in TMEM
  B_SFULL = B_QREADY + 1,     // both CTAs, per S buffer: S ready
  B_PFULL = B_SFULL + 2,      // rank 0: both CTAs' P(j) written (and O rescaled)
  B_PFREE = B_PFULL + 1,      // both CTAs: PV(j) done (O stable)
  B_ODONE = B_PFREE + 1,      // both CTAs: the last PV done
  B_DRAIN = B_ODONE + 1,
  NUM_BARS = B_DRAIN + 1
};
constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S = 0;    // S buffer b at COL_S + 128 b
constexpr uint32_t COL_O = 256;
constexpr uint32_t COL_Q = 384;  // Q as packed bf16 pairs (64 columns)
constexpr uint32_t IDESC_S = ptx::idesc_bf16(2 * BQ, BKV, 0);
constexpr uint32_t IDESC_PV = ptx::idesc_bf16(2 * BQ, D, 1);
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
constexpr int ARRIVALS = 2 * SOFTMAX_WARPS;  // per phase of the softmax-to-issuer barriers: both CTAs

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

// Max of 128 values as eight independent chains of three-input max.
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

// Pair MMA with A in tensor memory (each CTA's TMEM holds its 128 rows), B
// in shared memory (each CTA its half of N), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct Args {
  int n, heads, attn;   // attn = heads * 128
  const bf16* qkv;      // [n, 3 attn]
  bf16* out;            // [n, attn]
  float scale_log2;     // log2(e) / sqrt(128)
};

__global__ void __launch_bounds__(THREADS, 1)
    tc_attention_pair_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                             const Args args) {
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
  const uint32_t rank = cluster_rank();
  const int head = blockIdx.y;
  const int q0 = (int)(blockIdx.x >> 1) * 2 * BQ + (int)rank * BQ;  // this CTA's first query
  const int n = args.n;
  const int nkv = (n + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    mbar_init(bar(B_QREADY), ARRIVALS);
    mbar_init(bar(B_SFULL), 1);
    mbar_init(bar(B_SFULL + 1), 1);
    mbar_init(bar(B_PFULL), ARRIVALS);
    mbar_init(bar(B_PFREE), 1);
    mbar_init(bar(B_ODONE), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int cq = head * D, ck = args.attn + head * D, cv = 2 * args.attn + head * D;

  if (warp == 0) {
    if (lane == 0) {
      // producer: K(i) and V(i) halves into their rings, K first (needed a block earlier)
      const uint32_t kfull0 = peer_addr(bar(B_KFULL), 0u), vfull0 = peer_addr(bar(B_VFULL), 0u);
      bool ok = true;
      int last_k = -1, last_v = -1;
      for (int i = 0; i < nkv && ok; ++i) {
        const int s = i % NS;
        const uint32_t ph = (uint32_t)(i / NS) & 1u;
        if (!mbar_wait(bar(B_KEMPTY + s), ph ^ 1u, abort_flag)) { ok = false; break; }
        if (rank == 0) mbar_expect_tx(bar(B_KFULL + s), 2 * KH_BYTES);
        const uint32_t dk = base + OFF_K + s * KH_BYTES;
        const int krow = i * BKV + (int)rank * 64;
        tma_load_2d_pair(dk, &tmK, ck, krow, kfull0 + 8u * (uint32_t)s);
        tma_load_2d_pair(dk + KH_HALF, &tmK, ck + 64, krow, kfull0 + 8u * (uint32_t)s);
        last_k = i;
        if (!mbar_wait(bar(B_VEMPTY + s), ph ^ 1u, abort_flag)) { ok = false; break; }
        if (rank == 0) mbar_expect_tx(bar(B_VFULL + s), 2 * VH_BYTES);
        tma_load_2d_pair(base + OFF_V + s * VH_BYTES, &tmV, cv + (int)rank * 64, i * BKV, vfull0 + 8u * (uint32_t)s);
        last_v = i;
      }
      // on abort, let the newest copies land before the CTA can exit (rank 1
      // cannot observe rank 0's barriers; its copies finish within microseconds)
      if (!ok && (last_k >= 0 || last_v >= 0)) {
        if (rank == 0) {
          if (last_k >= 0) mbar_wait(bar(B_KFULL + last_k % NS), (uint32_t)(last_k / NS) & 1u, nullptr);
          if (last_v >= 0) mbar_wait(bar(B_VFULL + last_v % NS), (uint32_t)(last_v / NS) & 1u, nullptr);
        } else {
          spin_cycles(1LL << 22);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // pair MMA issuer
      const uint32_t peer_bar0 = peer_addr(bar0, 1u);
      auto commit_both = [&](int b) {
        tc_commit_pair(bar(b));
        tc_commit_pair(peer_bar0 + 8u * (uint32_t)b);
      };
      // descriptors: the address field holds (address >> 4), so a stage or a
      // K step further is the base descriptor plus (offset >> 4)
      const uint64_t dk = sw128_desc(base + OFF_K, 16, 1024), dv = sw128_desc(base + OFF_V, VH_BYTES, 1024);
      // S(j) = Q K_j^T into S buffer j % 2
      auto issue_s = [&](int j) {
        const uint64_t bk = dk + (uint64_t)(((j % NS) * KH_BYTES) >> 4);
        const uint32_t d = tmem + COL_S + (uint32_t)((j & 1) * BKV);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_ts_pair(d, tmem + COL_Q + (uint32_t)(k * 8),
                           bk + (uint64_t)(((k >> 2) * KH_HALF + (k & 3) * 32) >> 4), IDESC_S, k > 0 ? 1u : 0u);
      };
      // O += P(j) V_j, P(j) in the first 64 columns of S buffer j % 2
      auto issue_pv = [&](int j) {
        const uint64_t bv = dv + (uint64_t)(((j % NS) * VH_BYTES) >> 4);
        const uint32_t p = tmem + COL_S + (uint32_t)((j & 1) * BKV);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          mma_bf16_ts_pair(tmem + COL_O, p + (uint32_t)(k * 8), bv + (uint64_t)((k * 2048) >> 4), IDESC_PV,
                           (j > 0 || k > 0) ? 1u : 0u);
      };
      auto s_step = [&](int j) -> bool {  // K(j) landed -> S(j)
        if (!mbar_wait(bar(B_KFULL + j % NS), (uint32_t)(j / NS) & 1u, abort_flag)) return false;
        tc_fence_after();
        issue_s(j);
        commit_both(B_SFULL + (j & 1));
        commit_both(B_KEMPTY + j % NS);
        return true;
      };
      bool ok = nkv > 0 && mbar_wait(bar(B_QREADY), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        ok = s_step(0);
      }
      if (ok && nkv > 1) ok = s_step(1);
      for (int j = 0; j < nkv && ok; ++j) {
        if (!mbar_wait(bar(B_VFULL + j % NS), (uint32_t)(j / NS) & 1u, abort_flag)) { ok = false; break; }
        if (!mbar_wait(bar(B_PFULL), (uint32_t)j & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        issue_pv(j);
        commit_both(j + 1 < nkv ? B_PFREE : B_ODONE);
        commit_both(B_VEMPTY + j % NS);
        // S buffer j % 2 is free once PV(j) has read P(j) (the pipe runs in issue order)
        if (j + 2 < nkv && !s_step(j + 2)) { ok = false; break; }
      }
      // every MMA this thread issued has completed (and stopped reading both
      // CTAs' shared memory) once DRAIN flips
      tc_commit_pair(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, nullptr);
    }
  } else {
    // softmax warps 2-5: warp w owns TMEM lanes 32 (w % 4) .. +31; thread <-> query row r
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const uint32_t qready0 = peer_addr(bar(B_QREADY), 0u), pfull0 = peer_addr(bar(B_PFULL), 0u);
    const int row = q0 + r;
    // Q row into TMEM as packed bf16 pairs (the A-operand layout of the S MMA); rows past n are 0
    {
      uint32_t qv[64];
      if (row < n) {
        const uint4* src = reinterpret_cast<const uint4*>(args.qkv + (size_t)row * 3 * args.attn + cq);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint4 u = __ldg(src + i);
          qv[4 * i] = u.x;
          qv[4 * i + 1] = u.y;
          qv[4 * i + 2] = u.z;
          qv[4 * i + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) qv[i] = 0u;
      }
      tmem_st64(tmem + lane_addr + COL_Q, qv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(qready0);
    }
    const float sl2 = args.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    auto warp_wait = [&](int b, uint32_t parity) -> bool {
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait(bar(b), parity, abort_flag) ? 1 : 0;
      return __shfl_sync(0xffffffffu, w_ok, 0) != 0;
    };
    for (int j = 0; j < nkv; ++j) {
      const uint32_t s_col = COL_S + (uint32_t)((j & 1) * BKV);
      if (!warp_wait(B_SFULL + (j & 1), (uint32_t)(j >> 1) & 1u)) { ok = false; break; }
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
      // O is stable once PV(j-1) is done; only a rescale has to wait for it
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        if (!warp_wait(B_PFREE, (uint32_t)(j - 1) & 1u)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          const uint32_t ta = tmem + lane_addr + COL_O + (uint32_t)(c * 32);
          tmem_ld32(ta, o);
          uint32_t u[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(o[i] * corr);
          tmem_st32(ta, u);
        }
      }
      const f2_t scale2 = f2(sl2, sl2), negm2 = f2(-m_new, -m_new);
      f2_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[BKV / 2];
#pragma unroll
      for (int c = 0; c < BKV; c += 2) {
        float x0, x1;
        f2_split(f2_fma(f2(s[c], s[c + 1]), scale2, negm2), x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        acc[(c >> 1) & 3] = f2_add(acc[(c >> 1) & 3], f2(p0, p1));
        pk[c >> 1] = pack_bf16(p0, p1);
      }
      // P(j) over the first 64 columns of its S buffer
      tmem_st64(tmem + lane_addr + s_col, pk);
      float a0, a1;
      f2_split(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
      l = l * corr + (a0 + a1);
      m = m_new;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(pfull0);
    }
    if (ok && nkv > 0 && warp_wait(B_ODONE, 0u)) {
      tc_fence_after();
      const float inv = 1.0f / l;
      bf16* orow = args.out + (size_t)row * args.attn + head * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_addr + COL_O + (uint32_t)(c * 32), o);
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
  tc_fence_before();
  cluster_sync();  // no CTA leaves while its peer may still signal or read it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

}  // namespace attn2

// Rows from which attention uses the CTA-pair kernel (tuning knob, see
// fsdit_set_attention_pair_min_rows); below it the single-CTA kernel runs.
static int g_attn_pair_min_rows = 1 << 30;
int attention_pair_min_rows() { return g_attn_pair_min_rows; }

fsdit_status launch_attention_pair(const void* qkv, void* out, int n, int heads, int attn_w, cudaStream_t st) {
  using namespace attn2;
  if (((uintptr_t)qkv & 15u) != 0) {
    set_error("attention: qkv must be 16-byte aligned");
    return FSDIT_E_ALIGN;
  }
  static PerDevice<cudaError_t> attr;
  const cudaError_t attr_err = attr.get(
      [] {
        return cudaFuncSetAttribute(tc_attention_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    SMEM_BYTES);
      },
      cudaErrorInvalidDevice);
  if (attr_err != cudaSuccess) return cuda_check(attr_err, "cudaFuncSetAttribute(tc_attention_pair_kernel)");
  CUtensorMap tmK, tmV;
  FS_TRY(make_tmap_bf16(&tmK, qkv, (uint64_t)n, (uint64_t)3 * attn_w, (uint64_t)3 * attn_w, 64, 64));
  FS_TRY(make_tmap_bf16(&tmV, qkv, (uint64_t)n, (uint64_t)3 * attn_w, (uint64_t)3 * attn_w, 128, 64));
  Args a;
  a.n = n;
  a.heads = heads;
  a.attn = attn_w;
  a.qkv = reinterpret_cast<const bf16*>(qkv);
  a.out = reinterpret_cast<bf16*>(out);
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  const int nqb = (n + 2 * BQ - 1) / (2 * BQ);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * nqb, heads);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, tc_attention_pair_kernel, tmK, tmV, a), "tc_attention_pair_kernel");
}

}  // namespace fsdit

extern "C" fsdit_status fsdit_set_attention_pair_min_rows(int rows) {
  using namespace fsdit;
  if (rows < 1) {
    set_error("attention: the CTA-pair threshold must be at least 1 row");
    return FSDIT_E_SHAPE;
  }
  g_attn_pair_min_rows = rows;
  return FSDIT_OK;
}

extern "C" int fsdit_attention_pair_min_rows(void) { return fsdit::g_attn_pair_min_rows; }
