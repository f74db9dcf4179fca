// gqe_dispatch_noalloc: gqe_dispatch with its scratch in a fixed device array
// of this library instead of a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: their device memory is
// owned by another allocator (a serving runtime that reserves the whole GPU at
// start-up, or a plugin interface that passes the library only its input and
// output buffers), so they cannot call cudaMalloc, or any routine that
// allocates, for each call. This entry point serves them: the caller passes
// inputs and outputs only, and the dispatch scratch (per-token selection
// masks, per-tile counts and bases, the grouped-GEMM tile table and its
// length) lives in kScratchBytes of
// statically allocated device memory that every GPU loading the library holds
// until the process exits.
//
// Properties a caller must know:
//  - The first call on a device looks up the array's device address on that
//    device (cudaGetSymbolAddress, with the device current) and caches it;
//    make that first call before any stream capture. The cached address
//    belongs to that device's context: do not call this entry point again
//    after cudaDeviceReset (or any teardown of the primary context) in the
//    same process, since the library's module, and the array with it, may
//    then sit at another address.
//  - Every call on a device shares the one array, which keeps the last call's
//    contents. Each call writes every scratch word before reading it, so
//    nothing needs clearing, but calls that overlap on the GPU (different
//    streams, or threads with no ordering between them) race on the array.
//  - Configurations whose scratch exceeds kScratchBytes are rejected with
//    GQE_ERR_WORKSPACE before anything is launched.
#include <cuda_runtime.h>

#include "gqe_internal.h"

namespace gqe {
namespace noalloc_impl {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB per device
static __device__ __align__(256) unsigned char scratch[kScratchBytes];

// Device address of `scratch` in the current context, looked up on every
// call: a cached address would dangle after a device reset or a context
// re-creation in the same process.
void* scratch_address(cudaError_t* err) {
  void* p = nullptr;
  *err = cudaGetSymbolAddress(&p, scratch);
  return *err == cudaSuccess ? p : nullptr;
}

}  // namespace noalloc_impl
}  // namespace gqe

extern "C" gqe_status gqe_dispatch_noalloc(const gqe_config* cfg, const int32_t* idx,
                                           const gqe_bf16* x, const gqe_bf16* W_q,
                                           const gqe_bf16* W_qs, int32_t* counts, int32_t* offsets,
                                           int32_t* tok, int32_t* slot_pos, gqe_bf16* Qv,
                                           gqe_bf16* Qs, gqe_stream_t stream) {
  using namespace gqe;
  const size_t need = gqe_workspace_bytes(cfg, GQE_WS_DISPATCH);
  if (need == 0) return cfg == nullptr ? GQE_ERR_INVALID : check_cfg(cfg);
  if (need > noalloc_impl::kScratchBytes) return GQE_ERR_WORKSPACE;
  cudaError_t err = cudaSuccess;
  void* ws = noalloc_impl::scratch_address(&err);
  if (ws == nullptr) return GQE_ERR_CUDA;
  return gqe_dispatch(cfg, idx, x, W_q, W_qs, counts, offsets, tok, slot_pos, Qv, Qs, ws,
                      noalloc_impl::kScratchBytes, stream);
}
