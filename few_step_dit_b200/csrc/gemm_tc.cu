// Persistent bf16 GEMM on the sm_100a tensor cores: out = epi(A[M,K] B[N,K]^T).
//
// One CTA per SM (grid = min(tiles, SMs)), 192 threads in three roles:
//   warp 0  lane 0: TMA producer -- 128x64 A and 256x64 B tiles (128-byte
//           swizzle, no multicast) into a 4-stage shared-memory ring;
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
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(t_row + (uint32_t)(c * 32), v);
        const int col = nb * BN + c * 32;
        if (row < args.M && col < args.N) {
          if (col + 32 <= args.N) {
            epilogue_row<bf16, 32>(args.ep, row, col, v);
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

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;
static std::once_flag g_encode_once;

fsdit_status make_tmap_bf16(CUtensorMap* tm, const void* ptr, uint64_t rows, uint64_t cols, uint64_t row_stride_elems,
                            uint32_t box_rows, uint32_t box_cols) {
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

fsdit_status launch_linear_tc(const void* a, const void* w, const EpiParams& ep, int M, int N, int K,
                              cudaStream_t st) {
  using namespace gemm;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(tc_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
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
