// ffn_dense_noalloc: the dense FFN + residual add with its scratch memory in a
// fixed device array owned by the library instead of a caller workspace.
//
// For callers that cannot allocate device memory at the point of the call:
// code running inside a CUDA stream capture that must not add allocation
// nodes, runtimes whose memory is budgeted up front with no allocator handle
// to pass down, or plugins that only receive device pointers to inputs and
// outputs. They pass inputs and outputs; the scratch (gated activations and
// K-split partial sums of the down projection) lives in g_noalloc_scratch.
#include <cstdio>
#include <mutex>

#include "../../include/moeffn.h"
#include "common.cuh"

namespace moeffn {
int api_fail(int code, const char* msg);
}

namespace {

// Kept until the process exits on every GPU that loads the library.
constexpr size_t kNoAllocScratchBytes = MOEFFN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. On the host the
// array's name is only a stand-in, so the address is looked up once per
// device (with that device current) and cached.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return moeffn::api_fail(MOEFFN_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return moeffn::api_fail(MOEFFN_ERR_UNSUPPORTED, "ffn_dense_noalloc: device index");
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return moeffn::api_fail(MOEFFN_ERR_CUDA, "ffn_dense_noalloc: cudaGetSymbolAddress of the scratch array failed");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOEFFN_OK;
}

}  // namespace

extern "C" int ffn_dense_noalloc(const moeffn_ffn* w, const uint16_t* x, uint16_t* residual, int M, int act,
                                 moeffn_stream_t stream) {
  if (w == nullptr) return moeffn::api_fail(MOEFFN_ERR_INVALID, "ffn_dense_noalloc: null weights");
  if (M < 1) return moeffn::api_fail(MOEFFN_ERR_INVALID, "ffn_dense_noalloc: M < 1");
  const size_t need = moeffn_workspace_bytes(MOEFFN_KIND_DENSE, M, w->gate.cols, w->gate.rows, 0, 0);
  if (need == 0) return moeffn::api_fail(MOEFFN_ERR_INVALID, "ffn_dense_noalloc: bad shape");
  if (need > kNoAllocScratchBytes) {
    char msg[192];
    snprintf(msg, sizeof(msg),
             "ffn_dense_noalloc: this call needs %zu bytes of scratch, above the fixed %zu-byte array; "
             "use ffn_dense with a workspace",
             need, kNoAllocScratchBytes);
    return moeffn::api_fail(MOEFFN_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != MOEFFN_OK) return rc;
  // Nothing in this scratch has to start at zero: every byte read was written
  // earlier in the same call.
  return ffn_dense(w, x, residual, M, act, scratch, kNoAllocScratchBytes, stream);
}
