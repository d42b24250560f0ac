// mla_decode_attn_noalloc: mla_decode_attn whose workspace is a device array
// owned by the library, for callers that cannot allocate device memory.
//
// Who needs it: code that runs inside a host framework which owns every byte of
// device memory (an inference-server plugin or operator with a fixed memory
// budget, where only the framework may allocate), and latency-critical decode
// loops that must never call cudaMalloc, because cudaMalloc can synchronise the
// device and stall the other streams.  Such callers have no way to hand
// mla_decode_attn a workspace of their own.
//
// How: the split-KV partials live in one file-scope __device__ array of
// kNoAllocScratchBytes.  Every GPU that loads this library holds one copy of it
// until the process exits.  Host code cannot use the array's name as a device
// address (in host code it names a host-side stand-in), so the first call on each
// device looks the address up with cudaGetSymbolAddress while that device is
// current, and passes that address to the kernels.
#include <mutex>

#include "../../include/mla.h"
#include <cuda_runtime.h>

#include "decode.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB per device
constexpr int kMaxDevices = 64;

// The shared scratch.  Every call uses it; it keeps the previous call's contents.
__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::once_flag g_setup_once[kMaxDevices];
void* g_scratch_addr[kMaxDevices];
cudaError_t g_setup_error[kMaxDevices];   // outcome of the look-up, reported again on every later call

// Device address of g_decode_scratch on the current device (set-up on first use).
// A failed look-up is remembered for the device and reported (MLA_ERR_CUDA, with
// the CUDA error for mla_last_cuda_error) by every later call on it.
int scratch_on_current_device(void** addr) {
  int dev = 0;
  const cudaError_t eg = cudaGetDevice(&dev);
  if (eg != cudaSuccess) return mla::record_cuda_error(eg);
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::call_once(g_setup_once[dev], [dev] {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e == cudaSuccess && p == nullptr) e = cudaErrorInvalidSymbol;
    g_scratch_addr[dev] = (e == cudaSuccess) ? p : nullptr;
    g_setup_error[dev] = e;
  });
  *addr = g_scratch_addr[dev];
  return mla::record_cuda_error(g_setup_error[dev]);
}

}  // namespace

extern "C" int mla_decode_attn_noalloc(const mla_dims* dims, const mla_bf16* q_lat, const mla_bf16* pool,
                                       const int32_t* page_table, const int32_t* seq_lens, int32_t batch,
                                       int32_t nq, int32_t max_pages, int32_t num_pages, const mla_bf16* w_uv,
                                       mla_bf16* out, float* lse, int32_t* dev_status, void* stream) {
  void* scratch = nullptr;
  int st = scratch_on_current_device(&scratch);
  if (st != MLA_OK) return st;
  // Workspace this call would need; 0 means invalid arguments, which
  // mla_decode_attn below reports with the precise status.
  const size_t need = mla_decode_workspace_bytes(dims, batch, nq);
  if (need > kNoAllocScratchBytes) return MLA_ERR_WORKSPACE;
  // Nothing in the workspace has to start at zero: the split kernel writes every
  // partial before the combine kernel reads it.
  return mla_decode_attn(dims, q_lat, pool, page_table, seq_lens, batch, nq, max_pages, num_pages, w_uv,
                         scratch, kNoAllocScratchBytes, out, lse, dev_status, stream);
}
