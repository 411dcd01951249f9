// dit_block_forward_noalloc: the block forward for callers that cannot call
// cudaMalloc (or have torch allocate a workspace for them), e.g. a host
// application whose device memory is entirely owned by its own pool
// allocator, or a plain C caller that must not add allocations after start-up.
// The scratch the block needs (normalized operands, qkv, FFN hidden, and the
// compressed residual) lives in one file-scope device array instead of a
// caller-provided workspace.
#include <mutex>

#include "common.cuh"

namespace fsdit {

// Fixed size of the static scratch: 32 MiB.  It is part of the library's
// device image, so every GPU that loads libfsdit.so holds it until the
// process exits.
constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)32 << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of the array, looked up once per device (host code only
// sees a host-side stand-in under the array's name).
constexpr int NOALLOC_MAX_DEVICES = 64;
static void* g_noalloc_addr[NOALLOC_MAX_DEVICES] = {};
static std::mutex g_noalloc_mu;

static fsdit_status noalloc_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "cudaGetDevice");
  if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) {
    set_error("noalloc: device ordinal %d beyond the %d devices this entry point tracks", dev, NOALLOC_MAX_DEVICES);
    return FSDIT_E_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_check(e, "cudaGetSymbolAddress(noalloc scratch)");
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return FSDIT_OK;
}

}  // namespace fsdit

extern "C" fsdit_status dit_block_forward_noalloc(const fsdit_dims* dims, const fsdit_block_weights* w,
                                                  const fsdit_tokens* tok, const float* x_in, float* x_out,
                                                  fsdit_stream_t stream) {
  using namespace fsdit;
  FS_TRY(check_dims(dims));
  FS_TRY(check_block_weights(dims, w));
  FS_TRY(check_tokens(tok, false));
  // the scratch this block takes: the same carve as dit_block_forward, with
  // the block's real compressed row count
  const bool comp = tok->keep_idx != nullptr;
  Carve c{nullptr, 0};
  carve_block(c, dims, tok->n_tokens, comp ? n_compressed(tok) : tok->n_tokens, comp);
  if (c.off > NOALLOC_SCRATCH_BYTES) {
    set_error("noalloc: this block needs %zu bytes of scratch, more than the %zu-byte static array; "
              "use dit_block_forward with a caller-provided workspace",
              c.off, NOALLOC_SCRATCH_BYTES);
    return FSDIT_E_WORKSPACE;
  }
  // the array is looked up for the current device, so the stream must be one of its streams
  int cur = 0, sdev = 0;
  FS_TRY(cuda_check(cudaGetDevice(&cur), "cudaGetDevice"));
  FS_TRY(cuda_check(cudaStreamGetDevice((cudaStream_t)stream, &sdev), "cudaStreamGetDevice"));
  if (sdev != cur) {
    set_error("noalloc: the stream belongs to device %d but device %d is current; make the stream's device current",
              sdev, cur);
    return FSDIT_E_CUDA;
  }
  void* scratch = nullptr;
  FS_TRY(noalloc_scratch_address(&scratch));
  return dit_block_forward(dims, w, tok, x_in, x_out, scratch, NOALLOC_SCRATCH_BYTES, stream);
}
