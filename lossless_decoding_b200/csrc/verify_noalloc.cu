// uno_verify_block_noalloc: the block verifier for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain a workspace at the point of the call: a
// plug-in hosted by an inference engine that reserved all device memory for
// its own pool at start-up, code on a latency-critical path that cannot afford
// cudaMalloc (which may synchronise the device), or a caller from another
// language that has no device allocator at hand. This entry point gives them
// the verifier with its scratch in a fixed array that lives in the library's
// own device memory, so the call allocates nothing.
//
// The scratch is one file-scope array of kNoAllocScratchBytes per device. It
// is reserved on a device once the module that holds it is loaded there (with
// CUDA's default lazy loading: at this entry point's first use on that device)
// and stays reserved until the process exits. All calls on a device share it.
#include <atomic>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "uno.h"
#include "uno_host.h"

namespace {
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr int kMaxDevices = 64;
}  // namespace

// The scratch array. In host code this name is only a host-side stand-in:
// its device address must be looked up with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_verify_scratch[kNoAllocScratchBytes];

namespace {

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];  // device address of the array, per device

// Look up the array's device address for the current device (once per device).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return UNO_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return UNO_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_verify_scratch) != cudaSuccess || !ptr)
      return UNO_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return UNO_OK;
}

bool aligned_or_null(const void* p, uintptr_t a) { return uno_host::aligned(p, a); }

}  // namespace

extern "C" int uno_verify_block_noalloc(const void* p_logits, const void* q_logits,
                                        const int32_t* draft_tokens, int B, int K, int V,
                                        int dtype, uint64_t seed, uint64_t step,
                                        int32_t* out_tokens, int32_t* accepted_len,
                                        float* p_at_draft, float* q_at_draft, float* row_lse,
                                        void* stream) {
  if (dtype != UNO_BF16 && dtype != UNO_F32) return UNO_ERR_DTYPE;
  // Sizes are checked before B = 0 returns, exactly as uno_verify_block does
  // (the workspace size of one sequence is 0 only for bad K, V or dtype).
  if (B < 0 || B > (1 << 20) || uno_verify_workspace_bytes(1, K, V, dtype) == 0)
    return UNO_ERR_SIZE;
  if (B == 0) return UNO_OK;
  const size_t need = uno_verify_workspace_bytes(B, K, V, dtype);
  if (need == 0 || need > kNoAllocScratchBytes) return UNO_ERR_SIZE;  // beyond the fixed scratch
  // Check the caller's pointers before any work is queued.
  if (!p_logits || !q_logits || !draft_tokens || !out_tokens || !accepted_len)
    return UNO_ERR_NULL;
  if (!aligned_or_null(p_logits, 16) || !aligned_or_null(q_logits, 16) ||
      !aligned_or_null(draft_tokens, 4) || !aligned_or_null(out_tokens, 4) ||
      !aligned_or_null(accepted_len, 4) || !aligned_or_null(p_at_draft, 4) ||
      !aligned_or_null(q_at_draft, 4) || !aligned_or_null(row_lse, 4))
    return UNO_ERR_ALIGN;
  const int dev_status = uno_host::check_device();
  if (dev_status != UNO_OK) return dev_status;
  void* scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st != UNO_OK) return st;
  // The array keeps whatever the previous call left. uno_verify_block does
  // not depend on the contents of its workspace on entry (every counter and
  // record it reads is rewritten by the same call first), so nothing is cleared.
  return uno_verify_block(p_logits, q_logits, draft_tokens, B, K, V, dtype, seed, step,
                          out_tokens, accepted_len, p_at_draft, q_at_draft, row_lse, scratch,
                          kNoAllocScratchBytes, stream);
}
