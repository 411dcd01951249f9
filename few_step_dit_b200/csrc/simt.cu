// Exact-fp32 CUDA-core kernels (no TF32): the projection GEMM with the fused
// epilogues and joint attention.  They serve the fp32 configuration, whose
// parity bound (relative L2 1e-5) tensor-core inputs cannot meet.
#include <math.h>

#include "common.cuh"

namespace fsdit {

// ---------------------------------------------------------------- GEMM
// C[M,N] = A[M,K] B[N,K]^T, 64x64 tile, BK 16, 256 threads x (4 x 4) outputs.
constexpr int SG_BM = 64, SG_BN = 64, SG_BK = 16;

template <typename T>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const T* __restrict__ A, const T* __restrict__ B, int M,
                                                        int N, int K, EpiParams ep) {
  __shared__ float As[SG_BK][SG_BM + 4];
  __shared__ float Bs[SG_BK][SG_BN + 4];
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  const int m0 = blockIdx.y * SG_BM, n0 = blockIdx.x * SG_BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += SG_BK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid + i * 256;  // 0..1023
      const int r = e / SG_BK, kk = e % SG_BK;
      const int gm = m0 + r, gn = n0 + r, gk = k0 + kk;
      As[kk][r] = (gm < M && gk < K) ? ld_f32<T>(A + (size_t)gm * K + gk) : 0.f;
      Bs[kk][r] = (gn < N && gk < K) ? ld_f32<T>(B + (size_t)gn * K + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int col = n0 + tx * 4;
  if (col >= N) return;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = m0 + ty * 4 + i;
    if (row < M) epilogue_row<T, 4>(ep, row, col, acc[i]);
  }
}

fsdit_status launch_linear_simt(int dtype, const void* a, const void* w, const EpiParams& ep, int M, int N, int K,
                                cudaStream_t st) {
  dim3 grid((N + SG_BN - 1) / SG_BN, (M + SG_BM - 1) / SG_BM);
  if (dtype == FSDIT_BF16)
    simt_gemm_kernel<bf16><<<grid, 256, 0, st>>>((const bf16*)a, (const bf16*)w, M, N, K, ep);
  else
    simt_gemm_kernel<float><<<grid, 256, 0, st>>>((const float*)a, (const float*)w, M, N, K, ep);
  return cuda_check(cudaGetLastError(), "simt_gemm_kernel");
}

// ---------------------------------------------------------------- attention
// One warp per query row of one head; lane l holds channels [4l, 4l+4) of q
// (head_dim 128).  Keys and values of the head are staged 32 at a time in
// shared memory for the block's 8 warps; online softmax in fp32.
constexpr int SA_KEYS = 32;
template <typename T>
__global__ void __launch_bounds__(256) simt_attention_kernel(const T* __restrict__ qkv, T* __restrict__ out, int n,
                                                             int attn) {
  __shared__ float Ks[SA_KEYS][128];
  __shared__ float Vs[SA_KEYS][128];
  const int head = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q_row = blockIdx.x * 8 + warp;
  const size_t ld = (size_t)3 * attn;
  const float scale = rsqrtf(128.0f);
  float q[4], acc[4] = {0.f, 0.f, 0.f, 0.f};
  float m = -INFINITY, l = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    q[i] = (q_row < n) ? ld_f32<T>(qkv + (size_t)q_row * ld + head * 128 + lane * 4 + i) * scale : 0.f;
  for (int j0 = 0; j0 < n; j0 += SA_KEYS) {
    __syncthreads();
    for (int e = threadIdx.x; e < SA_KEYS * 128; e += blockDim.x) {
      const int r = e / 128, c = e % 128;
      const int j = j0 + r;
      Ks[r][c] = (j < n) ? ld_f32<T>(qkv + (size_t)j * ld + attn + head * 128 + c) : 0.f;
      Vs[r][c] = (j < n) ? ld_f32<T>(qkv + (size_t)j * ld + 2 * attn + head * 128 + c) : 0.f;
    }
    __syncthreads();
    const int nk = min(SA_KEYS, n - j0);
    for (int r = 0; r < nk; ++r) {
      float s = q[0] * Ks[r][lane * 4] + q[1] * Ks[r][lane * 4 + 1] + q[2] * Ks[r][lane * 4 + 2] +
                q[3] * Ks[r][lane * 4 + 3];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const float m_new = fmaxf(m, s);
      const float corr = expf(m - m_new);
      const float p = expf(s - m_new);
      l = l * corr + p;
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = acc[i] * corr + p * Vs[r][lane * 4 + i];
      m = m_new;
    }
  }
  if (q_row < n) {
    const float inv = 1.0f / l;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      out[(size_t)q_row * attn + head * 128 + lane * 4 + i] = cvt_from_f32<T>(acc[i] * inv);
  }
}

fsdit_status launch_attention_simt(int dtype, const void* qkv, void* out, int n, int heads, int attn,
                                   cudaStream_t st) {
  dim3 grid((n + 7) / 8, heads);
  if (dtype == FSDIT_BF16)
    simt_attention_kernel<bf16><<<grid, 256, 0, st>>>((const bf16*)qkv, (bf16*)out, n, attn);
  else
    simt_attention_kernel<float><<<grid, 256, 0, st>>>((const float*)qkv, (float*)out, n, attn);
  return cuda_check(cudaGetLastError(), "simt_attention_kernel");
}

}  // namespace fsdit
