// Decode step for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc, or any allocator, at
// the point where they run a decode step: serving engines that plan every
// device buffer once at start-up and forbid allocation afterwards, plugin
// hosts that hand a kernel library only the tensors of the call, and code
// that runs where no allocator is reachable.  They can still pass inputs and
// outputs, but not a workspace.  msa_sparse_attn_decode_noalloc runs the
// regular decode path with its scratch in a file-scope device array instead
// of a caller workspace.
//
// The array holds kNoAllocScratchBytes (16 MiB).  Every GPU that loads this
// library keeps that much device memory reserved for it until the process
// exits.  All calls on a device share the one array and it keeps the last
// call's contents, so two calls whose work overlaps on the GPU (different
// streams, or graphs replayed concurrently) race on it; callers must order
// such calls.  The status word at the start of the array is cleared on every
// call; nothing else in it needs to start at zero.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/msa.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// The array's device address belongs to the module as loaded in one CUDA
// context.  cudaDeviceReset destroys the device's primary context, and the
// next runtime call creates a new one with the module loaded again, possibly
// at another address; a caller running its own driver-API context on the
// device also sees its own copy.  So the address is cached per device
// together with the unique id of the context it was looked up in, and
// looked up again whenever the current context's id differs.
struct ScratchSlot {
  void *ptr = nullptr;
  unsigned long long ctx_id = 0;   // 0: not cached
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch[kMaxDevices];

// Device address of g_decode_scratch in the current context.  In host code
// the array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, called with the device current: once per device and
// context, then cached (see ScratchSlot).
int scratch_on_current_device(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    char m[256];
    snprintf(m, sizeof(m), "cudaGetDevice: %s", cudaGetErrorString(e));
    return msa::report_error(MSA_ERR_CUDA, m);
  }
  if (dev < 0 || dev >= kMaxDevices)
    return msa::report_error(MSA_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot &slot = g_scratch[dev];
  unsigned long long id = 0;
  if (slot.ptr && msa::current_context_id(&id) && id == slot.ctx_id) {
    *out = slot.ptr;
    return MSA_OK;
  }
  void *ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_decode_scratch);   // creates the context if there is none
  if (e != cudaSuccess || !ptr) {
    char m[256];
    snprintf(m, sizeof(m), "cudaGetSymbolAddress(decode scratch): %s", cudaGetErrorString(e));
    return msa::report_error(MSA_ERR_CUDA, m);
  }
  slot.ptr = ptr;
  slot.ctx_id = msa::current_context_id(&id) ? id : 0;   // 0: look it up again next call
  *out = ptr;
  return MSA_OK;
}

}  // namespace

extern "C" int msa_sparse_attn_decode_noalloc(const msa_params *p, const msa_bf16 *q,
                                              const msa_bf16 *q_idx, const msa_bf16 *k_cache,
                                              const msa_bf16 *v_cache, const msa_bf16 *k_idx_cache,
                                              const int32_t *seq_lens, msa_bf16 *out, int32_t *sel,
                                              msa_stream stream) {
  const size_t need = msa_workspace_bytes(p, MSA_OP_DECODE);
  if (need == 0)  // invalid params: the regular entry point reports the exact code
    return msa_sparse_attn_decode(p, q, q_idx, k_cache, v_cache, k_idx_cache, seq_lens, out, sel,
                                  nullptr, 0, stream);
  if (need > kNoAllocScratchBytes) {
    char m[256];
    snprintf(m, sizeof(m),
             "decode needs %zu bytes of scratch; the no-allocation entry point holds at most %zu "
             "(use msa_sparse_attn_decode with a workspace)",
             need, kNoAllocScratchBytes);
    return msa::report_error(MSA_ERR_WORKSPACE, m);
  }
  void *scratch = nullptr;
  int rc = scratch_on_current_device(&scratch);
  if (rc != MSA_OK) return rc;
  cudaError_t e = cudaMemsetAsync(scratch, 0, 256, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    char m[256];
    snprintf(m, sizeof(m), "clearing the scratch status word: %s", cudaGetErrorString(e));
    return msa::report_error(MSA_ERR_CUDA, m);
  }
  return msa_sparse_attn_decode(p, q, q_idx, k_cache, v_cache, k_idx_cache, seq_lens, out, sel,
                                scratch, kNoAllocScratchBytes, stream);
}
