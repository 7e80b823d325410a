// fa_noalloc.cu — the backward for callers that cannot allocate device memory.
//
// fa_bwd needs a caller-provided workspace (an fp32 dQ accumulator and the
// fp32 row terms D).  Some callers have no way to provide one: a plugin whose
// host engine owns and pre-reserves all of the GPU's memory and hands the
// plugin only its input and output buffers, or code that must not call
// cudaMalloc at all (it can synchronise the device, and it can fail under a
// fixed memory budget).  fa_bwd_noalloc serves them with a workspace that
// lives in this library's own static device memory: the array below, of
// FA_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds
// until the process exits.
//
// Contract, in short (the full text is in fa.h):
//   * nothing is allocated or freed — no cudaMalloc/cudaFree, no allocating
//     library routine;
//   * problems whose workspace exceeds FA_NOALLOC_SCRATCH_BYTES are rejected
//     with FA_ERR_UNSUPPORTED before anything is launched;
//   * every call on a device (in one CUDA context) shares the one array, which keeps the last
//     call's contents; the backward's first kernel zeroes what must start
//     at zero, so stale contents do no harm, but two calls whose kernels overlap
//     on the GPU (different streams, no ordering) race on the array;
//   * every call looks up the array's device address in the context current
//     on the calling thread: a __device__ array has one copy per CUDA context,
//     so an address cached per device ordinal would be wrong for a caller on a
//     non-primary context, or after cudaDeviceReset.  The first lookup in a
//     context may load the library's device code into it; make that first call
//     before any stream capture.
#include "../../include/fa.h"
#include "fa_internal.h"

namespace fa {

// The scratch itself.  In host code this name is only a host-side stand-in
// for the device array: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array in the calling thread's current context,
// or nullptr if the lookup fails.  Looked up on every call (cheap once the
// module is loaded), so it always belongs to the context the kernels run in.
static void* noalloc_scratch_for_current_context() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace fa

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                              int causal, const int32_t* cu_seqlens, int total_tokens, int dtype,
                              fa_stream_t stream) {
  const size_t need = fa_bwd_workspace_bytes(total_tokens, H, d);
  if (need == 0) return FA_ERR_INVALID_ARG;
  if (need > (size_t)FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;
  void* scratch = fa::noalloc_scratch_for_current_context();
  if (scratch == nullptr) return FA_ERR_CUDA;
  return fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, scratch,
                (size_t)FA_NOALLOC_SCRATCH_BYTES, stream);
}
