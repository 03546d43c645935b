// fa_noalloc.cu -- fa_bwd_noalloc: the backward for callers that cannot
// allocate device memory.
//
// fa_bwd needs a caller-provided workspace.  Some callers have no way to get
// one: a plugin or custom-op interface that hands the kernel only its input
// and output tensors, or code that must not allocate at that point (for
// instance while another component owns the allocator).  For them this entry
// point uses a fixed scratch array that lives in the library itself, so
// nothing is allocated per call.
//
// The scratch is a file-scope __device__ array of kScratchBytes; every GPU
// that loads the library holds it until the process exits.  Its device
// address is looked up once per device (cudaGetSymbolAddress, with that
// device current) on the first call made on that device.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/fa.h"

namespace {

constexpr size_t kScratchBytes = FA_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
std::mutex g_lock;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device, or null on failure.
// In host code the name g_scratch is only a host-side stand-in; the address
// a kernel can use must come from cudaGetSymbolAddress.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                              float scale, int causal, float dropout_p, uint64_t seed, void* stream) {
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return FA_OK;
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need == 0) return (d != 64 && d != 128) ? FA_ERR_UNSUPPORTED : FA_ERR_TOO_LARGE;
  if (need > kScratchBytes) return FA_ERR_TOO_LARGE;
  void* scratch = scratch_on_current_device();
  if (!scratch) return FA_ERR_CUDA;
  // The row pass zeroes the dQ accumulator and rewrites both row vectors, so
  // whatever an earlier call left in the scratch does not matter.
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, dropout_p, seed, scratch,
                kScratchBytes, stream);
}
