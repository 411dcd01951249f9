// Joint attention on the sm_100a tensor cores, CTA-pair form for long
// sequences (bf16 operands, fp32 softmax; same result as tc_attention_kernel).
//
// A cluster of two CTAs on neighbouring SMs takes 512 queries of one head as
// two 256-row pair tiles A and B; CTA rank r holds rows r*128 .. r*128+127 of
// each.  Every MMA is tcgen05.mma.cta_group::2 (M = 256) issued by one thread
// of rank 0:
//   S_t = Q_t K_j^T   N = 128 keys: rank r stages keys r*64 .. r*64+63 of
//                     block j (K-major), so each CTA loads half of K;
//   O_t += P_t V_j    N = 128 head columns: rank r stages columns
//                     r*64 .. r*64+63 of V_j for all 128 keys (MN-major),
//                     so each CTA loads half of V.
// Each CTA's TMEM holds S_A, S_B, O_A, O_B for its own 128 rows (512
// columns).  P is written by the softmax threads into shared memory (the
// halved K/V stages leave room for P_A and P_B), not over S: once a softmax
// warp has loaded its S_t(j) row into registers it signals the issuer, which
// computes S_t(j+1) while the exponentials of block j run.  The tensor pipe
// then alternates S(j+1) and PV(j) of both tiles with no softmax in between,
// instead of waiting, per tile, for softmax -> PV -> next S.
//
// Threads (320 per CTA): warp 0 lane 0 loads Q, K and V with TMA (each CTA
// its own halves; completion counted on rank 0's barriers); warp 1 allocates
// TMEM, and on rank 0 lane 0 issues the MMAs; warps 2-5 / 6-9 run the
// softmax of tile A / B, one thread per query row (TMEM lane): running max
// and sum in the log2 domain, O rescaled only when a row max grows by more
// than 8.  Every wait is bounded (see tc_ptx.cuh).
#include "tc_ptx.cuh"

namespace fsdit {
namespace attn2 {

constexpr int BQ = 128, BKV = 128, D = 128;
constexpr int QT_BYTES = 128 * 128 * 2;  // a 128-row Q or P tile: two 64-column swizzled boxes
constexpr int QT_HALF = QT_BYTES / 2;
constexpr int KH_BYTES = 64 * 128 * 2;   // this CTA's 64 keys x 128 columns: two 64-column boxes
constexpr int KH_HALF = KH_BYTES / 2;
constexpr int VH_BYTES = 128 * 64 * 2;   // 128 keys x this CTA's 64 columns: one box
constexpr int NS = 2;                    // K and V ring stages
constexpr int THREADS = 320;
constexpr int OFF_Q = 0;                    // Q_A, Q_B
constexpr int OFF_P = 2 * QT_BYTES;         // P_A, P_B
constexpr int OFF_K = 4 * QT_BYTES;         // K stage s at OFF_K + s * KH_BYTES
constexpr int OFF_V = OFF_K + NS * KH_BYTES;  // V stage s at OFF_V + s * VH_BYTES
constexpr int OFF_BAR = OFF_V + NS * VH_BYTES;
// barriers; the FULL ones and S_FREE / P_FULL are waited on in rank 0 only
enum {
  B_QFULL = 0,
  B_KFULL = 1,
  B_VFULL = B_KFULL + NS,
  B_KEMPTY = B_VFULL + NS,
  B_VEMPTY = B_KEMPTY + NS,
  B_SFULL = B_VEMPTY + NS,  // per tile, in both CTAs: S_t ready in TMEM
  B_SFREE = B_SFULL + 2,    // per tile, rank 0: both CTAs' S_t rows are in registers
  B_PFULL = B_SFREE + 2,    // per tile, rank 0: both CTAs' P_t written (and O_t rescaled)
  B_PFREE = B_PFULL + 2,    // per tile, in both CTAs: PV_t done (P_t free, O_t stable)
  B_ODONE = B_PFREE + 2,    // per tile, in both CTAs: the last PV_t done
  B_DRAIN = B_ODONE + 2,
  NUM_BARS = B_DRAIN + 1
};
constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_S = ptx::idesc_bf16(2 * BQ, BKV, 0);
constexpr uint32_t IDESC_PV = ptx::idesc_bf16(2 * BQ, D, 1);
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
constexpr int SOFTMAX_WARPS = 8;           // arrivals per tile barrier: 4 warps x 2 CTAs

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

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (the tensor core's operand reads), including reads issued by the
// peer CTA's MMA thread after the cluster-scope barrier arrive that follows.
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

struct Args {
  int n, heads, attn;  // attn = heads * 128
  bf16* out;           // [n, attn]
  float scale_log2;    // log2(e) / sqrt(128)
};

__global__ void __launch_bounds__(THREADS, 1)
    tc_attention_pair_kernel(const __grid_constant__ CUtensorMap tmQV, const __grid_constant__ CUtensorMap tmK,
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
  const int q0 = (int)(blockIdx.x >> 1) * 4 * BQ;  // first query of the cluster's 512
  const int n = args.n;
  const int nkv = (n + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(B_SFULL + t), 1);
      mbar_init(bar(B_SFREE + t), SOFTMAX_WARPS);
      mbar_init(bar(B_PFULL + t), SOFTMAX_WARPS);
      mbar_init(bar(B_PFREE + t), 1);
      mbar_init(bar(B_ODONE + t), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQV);
    prefetch_tmap(&tmK);
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
      // producer: Q once, then K(j+1) before V(j) (K is needed a block earlier)
      const uint32_t qfull0 = peer_addr(bar(B_QFULL), 0u);
      const uint32_t kfull0 = peer_addr(bar(B_KFULL), 0u), vfull0 = peer_addr(bar(B_VFULL), 0u);
      bool ok = true;
      if (rank == 0) mbar_expect_tx(bar(B_QFULL), 2 * 2 * QT_BYTES);
      for (int t = 0; t < 2; ++t) {
        const int row = q0 + t * 2 * BQ + (int)rank * BQ;
        tma_load_2d_pair(base + OFF_Q + t * QT_BYTES, &tmQV, cq, row, qfull0);
        tma_load_2d_pair(base + OFF_Q + t * QT_BYTES + QT_HALF, &tmQV, cq + 64, row, qfull0);
      }
      int last_k = -1, last_v = -1;
      auto load_k = [&](int i) -> bool {
        const int s = i % NS;
        const uint32_t ph = (uint32_t)(i / NS) & 1u;
        if (!mbar_wait(bar(B_KEMPTY + s), ph ^ 1u, abort_flag)) return false;
        if (rank == 0) mbar_expect_tx(bar(B_KFULL + s), 2 * KH_BYTES);
        const uint32_t dst = base + OFF_K + s * KH_BYTES;
        const int row = i * BKV + (int)rank * 64;
        tma_load_2d_pair(dst, &tmK, ck, row, kfull0 + 8u * (uint32_t)s);
        tma_load_2d_pair(dst + KH_HALF, &tmK, ck + 64, row, kfull0 + 8u * (uint32_t)s);
        last_k = i;
        return true;
      };
      auto load_v = [&](int i) -> bool {
        const int s = i % NS;
        const uint32_t ph = (uint32_t)(i / NS) & 1u;
        if (!mbar_wait(bar(B_VEMPTY + s), ph ^ 1u, abort_flag)) return false;
        if (rank == 0) mbar_expect_tx(bar(B_VFULL + s), 2 * VH_BYTES);
        tma_load_2d_pair(base + OFF_V + s * VH_BYTES, &tmQV, cv + (int)rank * 64, i * BKV,
                         vfull0 + 8u * (uint32_t)s);
        last_v = i;
        return true;
      };
      if (nkv > 0) ok = load_k(0);
      for (int j = 0; j < nkv && ok; ++j) {
        if (j + 1 < nkv && !load_k(j + 1)) { ok = false; break; }
        if (!load_v(j)) { ok = false; break; }
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
      // S_t(j) = Q_t K_j^T into TMEM columns 128t (each CTA: its 128 rows, all 128 keys)
      auto issue_s = [&](int t, int j) {
        const uint32_t sk = base + OFF_K + (j % NS) * KH_BYTES;
        const uint32_t sq = base + OFF_Q + t * QT_BYTES;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t oq = (uint32_t)((k >> 2) * QT_HALF + (k & 3) * 32);
          const uint32_t ok_ = (uint32_t)((k >> 2) * KH_HALF + (k & 3) * 32);
          mma_bf16_ss_pair(tmem + (uint32_t)(t * BKV), sw128_desc(sq + oq, 16, 1024), sw128_desc(sk + ok_, 16, 1024),
                           IDESC_S, k > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t(j) V_j (P_t in shared memory, K-major; V MN-major)
      auto issue_pv = [&](int t, int j) {
        const uint32_t sp = base + OFF_P + t * QT_BYTES;
        const uint32_t sv = base + OFF_V + (j % NS) * VH_BYTES;
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k) {
          const uint32_t op = (uint32_t)((k >> 2) * QT_HALF + (k & 3) * 32);
          mma_bf16_ss_pair(tmem + 256u + (uint32_t)(t * D), sw128_desc(sp + op, 16, 1024),
                           sw128_desc(sv + (uint32_t)(k * 2048), VH_BYTES, 1024), IDESC_PV,
                           (j > 0 || k > 0) ? 1u : 0u);
        }
      };
      bool ok = nkv > 0 && mbar_wait(bar(B_QFULL), 0, abort_flag);
      if (ok) ok = mbar_wait(bar(B_KFULL), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t) {
          issue_s(t, 0);
          commit_both(B_SFULL + t);
        }
        commit_both(B_KEMPTY);
      }
      for (int j = 0; j < nkv && ok; ++j) {
        if (j + 1 < nkv) {
          const int s1 = (j + 1) % NS;
          if (!mbar_wait(bar(B_KFULL + s1), (uint32_t)((j + 1) / NS) & 1u, abort_flag)) { ok = false; break; }
          for (int t = 0; t < 2 && ok; ++t) {
            if (!mbar_wait_cluster(bar(B_SFREE + t), (uint32_t)j & 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_s(t, j + 1);
            commit_both(B_SFULL + t);
          }
          if (!ok) break;
          commit_both(B_KEMPTY + s1);
        }
        const int s = j % NS;
        if (!mbar_wait(bar(B_VFULL + s), (uint32_t)(j / NS) & 1u, abort_flag)) { ok = false; break; }
        for (int t = 0; t < 2 && ok; ++t) {
          if (!mbar_wait_cluster(bar(B_PFULL + t), (uint32_t)j & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_pv(t, j);
          commit_both(j + 1 < nkv ? B_PFREE + t : B_ODONE + t);
        }
        if (!ok) break;
        commit_both(B_VEMPTY + s);
      }
      // every MMA this thread issued has completed (and stopped reading both
      // CTAs' shared memory) once DRAIN flips
      tc_commit_pair(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, nullptr);
    }
  } else {
    // softmax: tile t, thread <-> query row r of this CTA's half of the tile (TMEM lane r)
    const int t = (warp - 2) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const uint32_t s_col = (uint32_t)(t * BKV);
    const uint32_t o_col = 256u + (uint32_t)(t * D);
    const uint32_t p_row = base + OFF_P + (uint32_t)(t * QT_BYTES) + (uint32_t)(r * 128);
    const uint32_t swz = (uint32_t)(r & 7);
    const uint32_t sfree0 = peer_addr(bar(B_SFREE + t), 0u), pfull0 = peer_addr(bar(B_PFULL + t), 0u);
    const float sl2 = args.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // one lane waits on a barrier of this CTA, the warp follows
    auto warp_wait = [&](int b, uint32_t parity) -> bool {
      int w_ok = 1;
      if (lane == 0) w_ok = mbar_wait(bar(b), parity, abort_flag) ? 1 : 0;
      return __shfl_sync(0xffffffffu, w_ok, 0) != 0;
    };
    for (int j = 0; j < nkv; ++j) {
      if (!warp_wait(B_SFULL + t, (uint32_t)j & 1u)) { ok = false; break; }
      tc_fence_after();
      float s[BKV];
      tmem_ld128(tmem + lane_addr + s_col, s);
      // this warp's S rows are in registers: the issuer may overwrite S_t
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(sfree0);
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
      bool pv_done = j == 0;  // PV_t(j-1) has finished with P_t and O_t
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        if (!warp_wait(B_PFREE + t, (uint32_t)(j - 1) & 1u)) { ok = false; break; }
        pv_done = true;
        tc_fence_after();
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
      if (!pv_done && !warp_wait(B_PFREE + t, (uint32_t)(j - 1) & 1u)) { ok = false; break; }
      // P_t row r: keys 64b .. 64b+63 in box b, 16-byte chunk cc at (cc ^ (r & 7)) (128-byte swizzle)
#pragma unroll
      for (int b = 0; b < 2; ++b) {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const uint32_t* v = pk + b * 32 + cc * 4;
          st_shared_v4(p_row + (uint32_t)(b * QT_HALF) + (((uint32_t)cc ^ swz) << 4), v[0], v[1], v[2], v[3]);
        }
      }
      fence_proxy_async_all();
      float a0, a1;
      f2_split(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
      l = l * corr + (a0 + a1);
      m = m_new;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(pfull0);
    }
    if (ok && nkv > 0 && warp_wait(B_ODONE + t, 0u)) {
      tc_fence_after();
      const int row = q0 + t * 2 * BQ + (int)rank * BQ + r;
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
  static PerDevice<cudaError_t> attr;
  const cudaError_t attr_err = attr.get(
      [] {
        return cudaFuncSetAttribute(tc_attention_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    SMEM_BYTES);
      },
      cudaErrorInvalidDevice);
  if (attr_err != cudaSuccess) return cuda_check(attr_err, "cudaFuncSetAttribute(tc_attention_pair_kernel)");
  CUtensorMap tmQV, tmK;
  FS_TRY(make_tmap_bf16(&tmQV, qkv, (uint64_t)n, (uint64_t)3 * attn_w, (uint64_t)3 * attn_w, 128, 64));
  FS_TRY(make_tmap_bf16(&tmK, qkv, (uint64_t)n, (uint64_t)3 * attn_w, (uint64_t)3 * attn_w, 64, 64));
  Args a;
  a.n = n;
  a.heads = heads;
  a.attn = attn_w;
  a.out = reinterpret_cast<bf16*>(out);
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  const int nqb = (n + 4 * BQ - 1) / (4 * BQ);
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
  return cuda_check(cudaLaunchKernelEx(&cfg, tc_attention_pair_kernel, tmQV, tmK, a), "tc_attention_pair_kernel");
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
