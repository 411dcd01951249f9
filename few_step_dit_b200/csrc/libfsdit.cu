// Single translation unit of libfsdit.so: device globals (the error word) and
// every kernel live in one module, so no relocatable device code is needed.
#include "api.cu"
#include "elementwise.cu"
#include "fp8.cu"
#include "simt.cu"
#include "gemm_tc.cu"
#include "attn_tc.cu"
#include "attn_pair.cu"
#include "noalloc.cu"
#include "history.cu"
#include "decoder.cu"
#include "selfcheck.cu"
