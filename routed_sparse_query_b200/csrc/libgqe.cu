// Single translation unit of libgqe.so: the device status word and every
// kernel live in one module, so no relocatable device code is needed.
#include "router.cu"
#include "dispatch.cu"
#include "gemm.cu"
#include "attention.cu"
#include "decode.cu"
#include "api.cu"
#include "noalloc.cu"
#include "backward.cu"
#include "attn_bwd.cu"
