// Joint attention for bf16 operands.
#include "common.cuh"

namespace fsdit {

fsdit_status launch_attention_tc(const void* qkv, void* out, int n, int heads, int attn, cudaStream_t st) {
  return launch_attention_simt(FSDIT_BF16, qkv, out, n, heads, attn, st);
}

}  // namespace fsdit
