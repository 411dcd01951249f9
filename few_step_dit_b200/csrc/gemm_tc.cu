// Persistent bf16 GEMM on the sm_100a tensor cores: out = epi(A[M,K] B[N,K]^T).
//
// One CTA per SM (grid = min(tiles, SMs)), 192 threads in three roles:
//   warp 0  lane 0: TMA producer -- 128x64 A and 256x64 B tiles (128-byte
//           swizzle; each CTA loads only for itself) into a 4-stage ring;
//   warp 1  allocates 512 TMEM columns; lane 0 issues tcgen05.mma
//           (128x256x16, fp32 accumulators in TMEM, double-buffered) and
//           tcgen05.commit to release ring stages / publish accumulators;
//   warps 2-5: epilogue -- tcgen05.ld of the accumulator rows (warp w%4 owns
//           TMEM lanes 32*(w%4)..+31), fused bias / RoPE / GELU / residual,
//           16-byte stores; overlaps the next tile's main loop.
// Tiles are visited in bands of GROUP_N column tiles so the A rows and B
// columns that the 148 concurrent tiles touch stay resident in L2.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_ptx.cuh"

namespace fsdit {
namespace gemm {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int THREADS = 192;
constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + NUM_BARS * 8 + 16;
constexpr int GROUP_N = 16;
constexpr uint32_t IDESC = ptx::idesc_bf16(BM, BN, 0);

struct Args {
  int M, N, K;
  int tiles_m, tiles_n, group_n;
  EpiParams ep;
  // Tail cut (pair kernel only): tiles [0, full_units) run whole in the
  // first launch (n_units = full_units); every later tile is cut into
  // `split` units along K run by the SPLIT launch (n_units = cut tiles *
  // split; unit slot*split + s covers k-blocks [s*KB/split, (s+1)*KB/split)
  // of tile full_units + slot).  split == 1: no tail cut.
  int full_units, split, n_units;
  float* part;  // [slot*split + s][16 regions][4 chunks][8][32 lanes] float4 partial accumulators
  int* cnt;     // [slot][16 regions] arrivals, zero between launches
};

__device__ __forceinline__ void tile_coords(int tile, const Args& a, int& mb, int& nb) {
  const int per_group = a.group_n * a.tiles_m;
  const int g = tile / per_group;
  const int r = tile - g * per_group;
  const int n0 = g * a.group_n;
  const int gn = min(a.group_n, a.tiles_n - n0);
  mb = r / gn;
  nb = n0 + (r - mb * gn);
}

__global__ void __launch_bounds__(THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const Args args) {
  using namespace ptx;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bar0 = base + STAGES * STAGE_BYTES;
  // barrier ids: full[s] = s, empty[s] = STAGES+s, tfull[b] = 2S+b, tempty[b] = 2S+2+b, drain = 2S+4
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + STAGES * STAGE_BYTES + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar0 + 8 * s, 1);
      mbar_init(bar0 + 8 * (STAGES + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar0 + 8 * (2 * STAGES + b), 1);
      mbar_init(bar0 + 8 * (2 * STAGES + 2 + b), 128);
    }
    mbar_init(bar0 + 8 * (2 * STAGES + 4), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int num_tiles = args.tiles_m * args.tiles_n;
  const int KB = (args.K + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int last_s = -1;
      uint32_t last_ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, args, mb, nb);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar0 + 8 * (STAGES + s), ph ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = base + s * STAGE_BYTES;
          const uint32_t full = bar0 + 8 * s;
          mbar_expect_tx(full, STAGE_BYTES);
          tma_load_2d(sa, &tmA, kb * BK, mb * BM, full);
          tma_load_2d(sa + A_BYTES, &tmB, kb * BK, nb * BN, full);
          last_s = s;
          last_ph = ph;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      // on abort, let the newest copies land before the CTA can exit
      if (!ok && last_s >= 0) mbar_wait(bar0 + 8 * last_s, last_ph, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(bar0 + 8 * (2 * STAGES + 2 + buf), aph ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(bar0 + 8 * s, ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + s * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16_ss(d, sw128_desc(sa + 32 * k, 16, 1024), sw128_desc(sb + 32 * k, 16, 1024), IDESC,
                        (kb | k) != 0 ? 1u : 0u);
          tc_commit(bar0 + 8 * (STAGES + s));
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(bar0 + 8 * (2 * STAGES + buf));
      }
      // every MMA this thread issued has completed once `drain` flips
      tc_commit(bar0 + 8 * (2 * STAGES + 4));
      mbar_wait(bar0 + 8 * (2 * STAGES + 4), 0, nullptr);
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      int mb, nb;
      tile_coords(tile, args, mb, nb);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar0 + 8 * (2 * STAGES + buf), aph, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int row = mb * BM + q * 32 + lane;
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN);
      float ss = 0.0f;  // RESIDUAL producer: sum of out^2 over the current 128-column group
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(t_row + (uint32_t)(c * 32), v);
        const int col = nb * BN + c * 32;
        if (row < args.M && col < args.N) {
          if (col + 32 <= args.N) {
            ss += epilogue_row<bf16, 32>(args.ep, row, col, v);
            if ((c & 3) == 3 && args.ep.ss_part != nullptr) {
              args.ep.ss_part[(size_t)row * args.ep.ss_ld + (col >> 7)] = ss;
              ss = 0.0f;
            }
          } else {  // ragged last chunk (N % 32 != 0, N even)
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              if (col + i < args.N) epilogue_row<bf16, 2>(args.ep, row, col + i, v + i);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar0 + 8 * (2 * STAGES + 2 + buf));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm

// Pair-tile variant: a cluster of two CTAs computes a 256 x 256 output tile
// with tcgen05.mma.cta_group::2.  Each CTA stages only its own 128 A rows and
// 128 of the 256 B rows per K step, which halves the B operand's
// shared-memory and L2 traffic per FLOP.  A stage holds two 128-byte-wide
// boxes of each operand (64 KB per CTA, 3 stages): eight MMAs per barrier
// round trip.  Roles per CTA as above, but with eight epilogue warps (320
// threads: two per TMEM lane quarter, each on half the columns); warp 1 of
// CTA rank 0 issues the pair MMAs.  Both CTAs' TMA copies of a stage complete
// on rank 0's `full` barrier (rank 0 expects the bytes of both); the MMA
// commits release the stage in both CTAs.  Accumulator rows 0..127 of a tile
// sit in rank 0's TMEM, 128..255 in rank 1's; each CTA's epilogue stores its
// own rows and releases the accumulator buffer on rank 0's barrier (one arrive
// per warp).  An epilogue warp takes 32 x 32 blocks out of TMEM one row per
// lane and passes each through 4 KB of its own shared memory
// (warp_transpose32), so that every global access of the epilogue then covers
// four rows per instruction.  SPLIT = true instantiates the opt-in tail cut's second launch
// (units of K-slices of the last wave's tiles, see split_unit_epilogue).
namespace gemm2 {

// Tail cut bounds: at most SPLIT_MAX_UNITS partial units (256 KB of fp32
// partials each) and SPLIT_MAX_SLOTS cut tiles per launch.
constexpr int SPLIT_MAX_UNITS = 128, SPLIT_MAX_SLOTS = 64, SPLIT_REGIONS = 16;
constexpr int SPLIT_MIN_KB = 32, SPLIT_UNIT_KB = 12;

// Tile, k-block range, part and tail slot of work unit u: a whole tile
// (SPLIT = false: tile u) or part s of tail tile full_units + slot
// (SPLIT = true: k-blocks [s*KB/split, (s+1)*KB/split)).
template <bool SPLIT>
__device__ __forceinline__ void unit_work(int u, const gemm::Args& a, int KB, int& tile, int& kb0, int& kb1,
                                          int& s, int& slot) {
  if constexpr (!SPLIT) {
    tile = u;
    kb0 = 0;
    kb1 = KB;
    s = 0;
    slot = 0;
  } else {
    slot = u / a.split;
    s = u - slot * a.split;
    tile = a.full_units + slot;
    kb0 = s * KB / a.split;
    kb1 = (s + 1) * KB / a.split;
  }
}

constexpr int BM = 256, BN = 256, BK = 64;  // BK: bf16 elements per stage row (128 bytes)
constexpr int BK8 = 128;                     // E4M3 elements per stage row (128 bytes)
constexpr int HM = BM / 2, HN = BN / 2;  // per-CTA share of A rows and B rows
constexpr int STAGES = 3;
constexpr int BOXES = 2;  // 128-byte boxes per operand per stage
constexpr int A_BYTES = HM * BK * 2 * BOXES;
constexpr int B_BYTES = HN * BK * 2 * BOXES;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int EPI_WARPS = 8;  // two per TMEM lane quarter, each on half the columns
constexpr int THREADS = 64 + 32 * EPI_WARPS;
// barrier ids: full[s] = s (rank 0's counts both CTAs' copies), empty[s] = S+s,
// tfull[b] = 2S+b, tempty[b] = 2S+2+b (rank 0 only), drain = 2S+4
constexpr int NUM_BARS = 2 * STAGES + 5;
// after the ring: barriers, TMEM address and abort flag, then each epilogue
// warp's 4 KB block for warp_transpose32
constexpr int EPI_OFF = STAGES * STAGE_BYTES + 1024;
constexpr int SMEM_BYTES = EPI_OFF + EPI_WARPS * 4096 + 1024;
static_assert(NUM_BARS * 8 + 16 <= 1024, "barrier block");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
constexpr int GROUP_N = 8;
constexpr uint32_t IDESC = ptx::idesc_bf16(BM, BN, 0);
constexpr uint32_t IDESC_FP8 = ptx::idesc_e4m3(BM, BN);

// Epilogue of one split unit, for one epilogue warp's region (its rank's rows
// of one TMEM lane quarter, one column half): park this unit's fp32
// accumulators of the region in the scratch, release the TMEM buffer (arrive
// on `tempty`, rank 0's barrier: locally when `local`, else through the
// cluster), count the part in; the warp that brings the region's last part
// sums all parts in split order -- the same result whichever unit finishes
// last -- runs the epilogue and clears the counter for the next launch.
__device__ __forceinline__ void split_unit_epilogue(const gemm::Args& args, uint32_t t_row, int slot, int sp,
                                                 int region, int row, bool row_ok, int nb, int c0, int lane,
                                                 uint32_t tempty, bool local) {
  using namespace ptx;
  constexpr int CHUNKS = BN / 64;                 // 32-column chunks of a region
  constexpr int REGION_F4 = CHUNKS * 8 * 32;      // float4s of one region's part
  float4* mine = reinterpret_cast<float4*>(args.part) +
                 ((size_t)(slot * args.split + sp) * SPLIT_REGIONS + region) * REGION_F4;
#pragma unroll 1
  for (int c = 0; c < CHUNKS; ++c) {
    float v[32];
    tmem_ld32(t_row + (uint32_t)((c0 + c) * 32), v);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      mine[(c * 8 + i) * 32 + lane] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) {
    if (local) mbar_arrive(tempty);
    else mbar_arrive_cluster(tempty);
  }
  __threadfence();
  __syncwarp();
  int last = 0;
  int* cnt = args.cnt + slot * SPLIT_REGIONS + region;
  if (lane == 0) last = atomicAdd(cnt, 1) == args.split - 1 ? 1 : 0;
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();
  const float4* parts = reinterpret_cast<const float4*>(args.part) +
                        ((size_t)(slot * args.split) * SPLIT_REGIONS + region) * REGION_F4;
#pragma unroll 1
  for (int c = 0; c < CHUNKS; ++c) {
    const int col = nb * BN + (c0 + c) * 32;
    const bool full = row_ok && col + 32 <= args.N;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0.f;
#pragma unroll 1
    for (int p = 0; p < args.split; ++p) {
      const float4* src = parts + (size_t)p * SPLIT_REGIONS * REGION_F4 + c * 8 * 32 + lane;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 t = __ldcg(src + i * 32);
        v[4 * i] += t.x;
        v[4 * i + 1] += t.y;
        v[4 * i + 2] += t.z;
        v[4 * i + 3] += t.w;
      }
    }
    if (full) {
      Epi32Pre pre;
      epi32_prefetch(args.ep, row, col, pre);
      epi32_apply(args.ep, row, col, v, pre);
    } else if (row_ok && col < args.N) {
#pragma unroll
      for (int i = 0; i < 32; i += 2)
        if (col + i < args.N) epilogue_row<bf16, 2>(args.ep, row, col + i, v + i);
    }
  }
  if (lane == 0) *cnt = 0;
}

// FP8 = true: E4M3 operands (kind::f8f6f4, 32 K elements per MMA), the same
// 128-byte stage rows; the epilogue applies the per-row / per-column scales.
template <bool FP8, bool SPLIT>
__global__ void __launch_bounds__(THREADS, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const gemm::Args args) {
  constexpr int BKE = (FP8 ? BK8 : BK) * BOXES;  // K elements per stage
  constexpr int BOXE = FP8 ? BK8 : BK;          // K elements per box
  using namespace ptx;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bar0 = base + STAGES * STAGE_BYTES;
  auto FULL = [&](int s) { return bar0 + 8u * (uint32_t)s; };
  auto EMPTY = [&](int s) { return bar0 + 8u * (uint32_t)(STAGES + s); };
  auto TFULL = [&](int b) { return bar0 + 8u * (uint32_t)(2 * STAGES + b); };
  auto TEMPTY = [&](int b) { return bar0 + 8u * (uint32_t)(2 * STAGES + 2 + b); };
  const uint32_t DRAIN = bar0 + 8u * (uint32_t)(2 * STAGES + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + STAGES * STAGE_BYTES + NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int cid = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(FULL(s), 1);
      mbar_init(EMPTY(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(TFULL(b), 1);
      mbar_init(TEMPTY(b), 2 * EPI_WARPS);  // epilogue warps of both CTAs
    }
    mbar_init(DRAIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int KB = (args.K + BKE - 1) / BKE;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int last_s = -1;
      uint32_t last_ph = 0;
      bool ok = true;
      const uint32_t full0 = peer_addr(FULL(0), 0u);  // rank 0's full barriers
      for (int u = cid; u < args.n_units && ok; u += ncl) {
        int tile, kb0, kb1, sp, slot, mb, nb;
        unit_work<SPLIT>(u, args, KB, tile, kb0, kb1, sp, slot);
        gemm::tile_coords(tile, args, mb, nb);
        const int row_a = mb * BM + (int)rank * HM, row_b = nb * BN + (int)rank * HN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(EMPTY(s), ph ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = base + s * STAGE_BYTES;
          const uint32_t full = full0 + 8u * (uint32_t)s;
          if (rank == 0) mbar_expect_tx(FULL(s), 2 * STAGE_BYTES);
          for (int bx = 0; bx < BOXES; ++bx) {
            tma_load_2d_pair(sa + bx * (HM * 128), &tmA, kb * BKE + bx * BOXE, row_a, full);
            tma_load_2d_pair(sa + A_BYTES + bx * (HN * 128), &tmB, kb * BKE + bx * BOXE, row_b, full);
          }
          last_s = s;
          last_ph = ph;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      // on abort, let the newest copies land before the CTA can exit (rank 1
      // cannot observe rank 0's barrier; its copies finish within microseconds)
      if (!ok && last_s >= 0) {
        if (rank == 0) mbar_wait(FULL(last_s), last_ph, nullptr);
        else spin_cycles(1LL << 22);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // pair MMA issuer
      const uint32_t empty_peer0 = peer_addr(EMPTY(0), 1u), tfull_peer0 = peer_addr(TFULL(0), 1u);
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      bool ok = true;
      for (int u = cid; u < args.n_units && ok; u += ncl, ++it) {
        int tile, kb0, kb1, sp, slot;
        unit_work<SPLIT>(u, args, KB, tile, kb0, kb1, sp, slot);
        const int buf = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait_cluster(TEMPTY(buf), aph ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(FULL(s), ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + s * STAGE_BYTES, sb = sa + A_BYTES;
          // eight MMAs of 32 bytes of K each (16 bf16 or 32 E4M3 elements), four per box
#pragma unroll
          for (int k = 0; k < 4 * BOXES; ++k) {
            const uint32_t oa = (uint32_t)((k >> 2) * (HM * 128) + (k & 3) * 32);
            const uint32_t ob = (uint32_t)((k >> 2) * (HN * 128) + (k & 3) * 32);
            const uint32_t acc = (kb != kb0 || k != 0) ? 1u : 0u;
            if constexpr (FP8)
              mma_e4m3_ss_pair(d, sw128_desc(sa + oa, 16, 1024), sw128_desc(sb + ob, 16, 1024), IDESC_FP8, acc);
            else
              mma_bf16_ss_pair(d, sw128_desc(sa + oa, 16, 1024), sw128_desc(sb + ob, 16, 1024), IDESC, acc);
          }
          tc_commit_pair(EMPTY(s));
          tc_commit_pair(empty_peer0 + 8u * (uint32_t)s);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(TFULL(buf));
        tc_commit_pair(tfull_peer0 + 8u * (uint32_t)buf);
      }
      // every MMA this thread issued has completed (and stopped reading both
      // CTAs' shared memory) once `drain` flips
      tc_commit_pair(DRAIN);
      mbar_wait(DRAIN, 0, nullptr);
    }
  } else {
    const int q = warp & 3;                    // TMEM lane quarter this warp may access
    const int c0 = ((warp - 2) >> 2) * (BN / 64);  // first of its BN/64 column chunks
    const uint32_t tempty0 = peer_addr(TEMPTY(0), 0u);
    // this warp's region of a tile: its rank's rows of lane quarter q, its
    // column half (the unit of the split-tail bookkeeping)
    const int region = ((int)rank * 4 + q) * 2 + (c0 != 0 ? 1 : 0);
    float4* epi_buf = reinterpret_cast<float4*>(base_ptr + EPI_OFF) + (warp - 2) * 256;
    int it = 0;
    for (int u = cid; u < args.n_units; u += ncl, ++it) {
      int tile, kb0, kb1, sp, slot;
      unit_work<SPLIT>(u, args, KB, tile, kb0, kb1, sp, slot);
      const int buf = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      int mb, nb;
      gemm::tile_coords(tile, args, mb, nb);
      const int row = mb * BM + (int)rank * HM + q * 32 + lane;
      const bool row_ok = row < args.M;
      // RMSNorm consumer: 1/rms of this lane's row, read while the tile's
      // accumulators are still being computed
      const float lane_rstd = !SPLIT && args.ep.norm_ss != nullptr && row_ok ? norm_rstd(args.ep, row) : 0.0f;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(TFULL(buf), aph, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN);
      if constexpr (SPLIT) {
        split_unit_epilogue(args, t_row, slot, sp, region, row, row_ok, nb, c0, lane,
                            rank == 0 ? TEMPTY(buf) : tempty0 + 8u * (uint32_t)buf, rank == 0);
        continue;
      }
      const int row0 = row - lane;  // first row of this warp's 32 x 32 blocks
      float ssq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // RESIDUAL producer: rows row0 + lane/8 + 4i
#pragma unroll 1
      for (int c = c0; c < c0 + BN / 64; ++c) {
        const int col = nb * BN + c * 32;
        float v[32];
        if (col + 32 <= args.N) {  // warp-uniform: the block's columns are all inside
          EpiTPre pre;
          epiT_prefetch(args.ep, row0, col, args.M, lane, pre, lane_rstd);
          tmem_ld32(t_row + (uint32_t)(c * 32), v);
          float w[32];
          warp_transpose32(epi_buf, v, w, lane);
          epiT_apply(args.ep, row0, col, args.M, lane, w, pre, ssq);
        } else {
          tmem_ld32(t_row + (uint32_t)(c * 32), v);
          if (row_ok && col < args.N) {  // ragged last chunk (N % 32 != 0, N even)
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              if (col + i < args.N) epilogue_row<bf16, 2>(args.ep, row, col + i, v + i);
          }
        }
      }
      if (args.ep.ss_part != nullptr && nb * BN + c0 * 32 < args.N) {
        // the eight lanes of a row hold 4 columns each of the warp's 128: sum
        // them (fixed order) and store the row's partial for this group (a
        // warp whose columns lie past N -- the last tile of an N that is an
        // odd multiple of 128 -- has no group)
        const int grp = (nb * BN + c0 * 32) >> 7;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float t = ssq[i];
          t += __shfl_xor_sync(0xffffffffu, t, 1);
          t += __shfl_xor_sync(0xffffffffu, t, 2);
          t += __shfl_xor_sync(0xffffffffu, t, 4);
          const int r = row0 + (lane >> 3) + 4 * i;
          if ((lane & 7) == 0 && r < args.M) args.ep.ss_part[(size_t)r * args.ep.ss_ld + grp] = t;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(TEMPTY(buf));
        else mbar_arrive_cluster(tempty0 + 8u * (uint32_t)buf);
      }
    }
  }
  tc_fence_before();
  cluster_sync();  // no CTA leaves while its peer may still signal or read it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm2

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;
static std::once_flag g_encode_once;

// The driver's cuTensorMapEncodeTiled, looked up once.
static fsdit_status encode_fn() {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (g_encode_tiled == nullptr) {
    set_error("cuTensorMapEncodeTiled is not available from the driver");
    return FSDIT_E_CUDA;
  }
  return FSDIT_OK;
}

fsdit_status make_tmap_bf16(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t cols, uint64_t row_stride_elems,
                            uint32_t box_rows, uint32_t box_cols) {
  FS_TRY(encode_fn());
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(row_stride_elems * 2)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode_tiled(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (%d) rows=%llu cols=%llu", (int)r, (unsigned long long)rows,
              (unsigned long long)cols);
    return FSDIT_E_CUDA;
  }
  return FSDIT_OK;
}

// How many CTA pairs of tc_gemm_pair_kernel fit on the device at once
// (0: the pair kernel cannot run, use the single-CTA kernel).
fsdit_status make_tmap_u8(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t cols, uint64_t row_stride,
                          uint32_t box_rows, uint32_t box_cols) {
  FS_TRY(encode_fn());
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode_tiled(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled (u8) failed (%d) rows=%llu cols=%llu", (int)r, (unsigned long long)rows,
              (unsigned long long)cols);
    return FSDIT_E_CUDA;
  }
  return FSDIT_OK;
}

static int pair_clusters_resident() {
  static PerDevice<int> resident;
  return resident.get([] {
    int n = 0;
    for (auto fn : {gemm2::tc_gemm_pair_kernel<false, false>, gemm2::tc_gemm_pair_kernel<true, false>,
                    gemm2::tc_gemm_pair_kernel<false, true>, gemm2::tc_gemm_pair_kernel<true, true>}) {
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm2::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 0) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
      }
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * 74);
    cfg.blockDim = dim3(gemm2::THREADS);
    cfg.dynamicSmemBytes = gemm2::SMEM_BYTES;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, gemm2::tc_gemm_pair_kernel<false, false>, &cfg) == cudaSuccess) n = c;
    (void)cudaGetLastError();
    return n;
  }, 0);
}

static fsdit_status launch_linear_pair(const void* a, const void* w, const EpiParams& ep, int M, int N, int K,
                                       int clusters, bool fp8, cudaStream_t st) {
  using namespace gemm2;
  CUtensorMap tmA, tmB;
  fsdit_status s = fp8 ? make_tmap_u8(&tmA, a, (uint64_t)M, (uint64_t)K, (uint64_t)K, HM, BK8)
                       : make_tmap_bf16(&tmA, a, (uint64_t)M, (uint64_t)K, (uint64_t)K, HM, BK);
  if (s != FSDIT_OK) return s;
  s = fp8 ? make_tmap_u8(&tmB, w, (uint64_t)N, (uint64_t)K, (uint64_t)K, HN, BK8)
          : make_tmap_bf16(&tmB, w, (uint64_t)N, (uint64_t)K, (uint64_t)K, HN, BK);
  if (s != FSDIT_OK) return s;
  gemm::Args args;
  args.M = M;
  args.N = N;
  args.K = K;
  args.tiles_m = (M + BM - 1) / BM;
  args.tiles_n = (N + BN - 1) / BN;
  args.group_n = GROUP_N < args.tiles_n ? GROUP_N : args.tiles_n;
  args.ep = ep;
  const int tiles = args.tiles_m * args.tiles_n;
  // Tail cut: the R tiles of a partial last wave leave most CTA pairs idle;
  // cut each into S units along K (S <= pairs / R) that run as a second
  // launch of the SPLIT kernel, so the last wave is about 1/S of a tile
  // long.  The whole tiles run in the first launch, whose kernel has no split
  // code.  Only long K pays for the second launch and the fixup: at least
  // SPLIT_MIN_KB k-blocks per tile and SPLIT_UNIT_KB per unit.
  const int KB = (K + (fp8 ? BK8 : BK) * BOXES - 1) / ((fp8 ? BK8 : BK) * BOXES);
  int R = 0, S = 1;
  if (ep.split_part != nullptr && ep.split_cnt != nullptr && KB >= SPLIT_MIN_KB) {
    R = tiles % clusters;
    S = R > 0 ? clusters / R : 1;
    if (S > KB / SPLIT_UNIT_KB) S = KB / SPLIT_UNIT_KB;
    if (S > 8) S = 8;
    if (R > 0 && R * S > SPLIT_MAX_UNITS) S = SPLIT_MAX_UNITS / R;
    if (R == 0 || R > SPLIT_MAX_SLOTS || S < 2) {
      R = 0;
      S = 1;
    }
  }
  args.full_units = tiles - R;
  args.split = S;
  args.part = ep.split_part;
  args.cnt = ep.split_cnt;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  auto launch = [&](bool split, int units) -> fsdit_status {
    args.n_units = units;
    const int ncl = units < clusters ? units : clusters;
    cfg.gridDim = dim3(2 * ncl);
    cudaError_t e;
    if (fp8)
      e = split ? cudaLaunchKernelEx(&cfg, tc_gemm_pair_kernel<true, true>, tmA, tmB, args)
                : cudaLaunchKernelEx(&cfg, tc_gemm_pair_kernel<true, false>, tmA, tmB, args);
    else
      e = split ? cudaLaunchKernelEx(&cfg, tc_gemm_pair_kernel<false, true>, tmA, tmB, args)
                : cudaLaunchKernelEx(&cfg, tc_gemm_pair_kernel<false, false>, tmA, tmB, args);
    return cuda_check(e, split ? "tc_gemm_pair_kernel (tail cut)" : "tc_gemm_pair_kernel");
  };
  if (args.full_units > 0) FS_TRY(launch(false, args.full_units));
  if (R > 0) {
    FS_TRY(launch(true, R * S));
    if (args.full_units > 0) prof_add_kernels(1);
  }
  return FSDIT_OK;
}

// E4M3 projection: always on pair tiles (their epilogue applies the scales).
fsdit_status launch_linear_fp8_tc(const uint8_t* qa, const uint8_t* qw, const EpiParams& ep, int M, int N, int K,
                                  cudaStream_t st) {
  const int clusters = pair_clusters_resident();
  if (clusters <= 0) {
    set_error("linear_fp8: the CTA-pair GEMM cannot be made resident on this device");
    return FSDIT_E_CUDA;
  }
  return launch_linear_pair(qa, qw, ep, M, N, K, clusters, true, st);
}

fsdit_status launch_linear_tc(const void* a, const void* w, const EpiParams& ep, int M, int N, int K,
                              cudaStream_t st) {
  // pair tiles once there are two 128-row blocks to share them; their
  // epilogue moves bias, output, residual and RoPE table in 16-byte pieces
  auto a16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
  const bool f32_out = ep.epi == FSDIT_EPI_RESIDUAL || ep.epi == FSDIT_EPI_BIAS_F32 || ep.epi == EPI_UNPATCH;
  const bool vec_ok = a16(ep.bias) && a16(ep.out) && ep.ldo % (f32_out ? 4 : 8) == 0 &&
                      (ep.epi != EPI_UNPATCH || ep.up_ps % 4 == 0) &&
                      (ep.epi != FSDIT_EPI_RESIDUAL || (a16(ep.resid) && ep.ldr % 4 == 0)) &&
                      (ep.rope_cs == nullptr || a16(ep.rope_cs)) && (ep.head_dim & (ep.head_dim - 1)) == 0;
  if (M > gemm2::HM && vec_ok) {
    const int clusters = pair_clusters_resident();
    if (clusters > 0) return launch_linear_pair(a, w, ep, M, N, K, clusters, false, st);
  }
  using namespace gemm;
  static PerDevice<cudaError_t> attr;
  const cudaError_t attr_err = attr.get(
      [] { return cudaFuncSetAttribute(tc_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES); },
      cudaErrorInvalidDevice);
  if (attr_err != cudaSuccess) return cuda_check(attr_err, "cudaFuncSetAttribute(tc_gemm_kernel)");
  CUtensorMap tmA, tmB;
  fsdit_status s = make_tmap_bf16(&tmA, a, (uint64_t)M, (uint64_t)K, (uint64_t)K, BM, BK);
  if (s != FSDIT_OK) return s;
  s = make_tmap_bf16(&tmB, w, (uint64_t)N, (uint64_t)K, (uint64_t)K, BN, BK);
  if (s != FSDIT_OK) return s;
  Args args;
  args.M = M;
  args.N = N;
  args.K = K;
  args.tiles_m = (M + BM - 1) / BM;
  args.tiles_n = (N + BN - 1) / BN;
  args.group_n = GROUP_N < args.tiles_n ? GROUP_N : args.tiles_n;
  args.ep = ep;
  const int tiles = args.tiles_m * args.tiles_n;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  tc_gemm_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tmA, tmB, args);
  return cuda_check(cudaGetLastError(), "tc_gemm_kernel");
}

}  // namespace fsdit
