// bc_gemv_noalloc: the column-gathered GEMV for callers that cannot hand the
// library a scratch buffer.
//
// bc_gemv needs scratch device memory for its split-K partial sums and the
// tickets that elect the CTA which reduces them.  Some callers cannot
// allocate that memory: an operator plugged into another framework whose
// allocator owns all device memory and exposes only the operator's inputs and
// outputs, or a caller that must not call cudaMalloc on its serving path
// because cudaMalloc can synchronise the device and stall every stream.  This
// entry point keeps the scratch in a file-scope __device__ array instead, so
// the caller passes only W, x, the channel list and y.
//
// The array holds kNoAllocMaxDout * 256 bytes + the tickets (8 MiB + 1 KiB)
// and lives on every GPU that loads the library until the process exits.
// Its device address is looked up once per device, on the first call made
// while that device is current; make that first call before capturing a
// stream into a CUDA graph.  All calls share the one array and it keeps the
// last call's contents: the tickets are cleared on every call, and calls that
// overlap on the GPU (different streams, or different host threads on the
// same device) race on it and must be serialised by the caller.
#include "../../include/bytecross.h"
#include "common.cuh"
#include "kernels.h"

#include <stdio.h>
#include <mutex>

namespace {

constexpr int kNoAllocMaxDout = 32768;
constexpr size_t kPartialBytes = 4ull * bc::kGemvMaxContrib * kNoAllocMaxDout;
constexpr size_t kTicketBytes = 4ull * (kNoAllocMaxDout / 128);   // one ticket per 128-column tile

static __device__ __align__(256) unsigned char g_scratch[kPartialBytes + kTicketBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (host code may not use
// the symbol itself: on the host it names a stand-in, not device memory).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" int bc_gemv_noalloc_max_dout(void) { return kNoAllocMaxDout; }

extern "C" bc_status bc_gemv_noalloc(const void* W, int d_in, int d_out, const float* x, const int* idx,
                                     int k, float* y, void* stream) {
  if (d_out > kNoAllocMaxDout) {
    char msg[160];
    snprintf(msg, sizeof msg, "bc_gemv_noalloc: d_out %d exceeds the built-in scratch maximum of %d columns",
             d_out, kNoAllocMaxDout);
    bc::set_error(msg);
    return BC_EINVAL;
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    bc::set_error("bc_gemv_noalloc: looking up the scratch array's device address failed");
    return BC_ECUDA;
  }
  if (d_out > 0 && d_out % bc::kColTile == 0) {
    // the tickets must start at zero; a failed earlier call may have left some set
    const size_t part = (4ull * bc::kGemvMaxContrib * d_out + 255) & ~size_t(255);
    e = cudaMemsetAsync(static_cast<char*>(scratch) + part, 0, 4ull * (d_out / 128),
                        static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
      bc::set_error("bc_gemv_noalloc: clearing the tickets failed");
      return BC_ECUDA;
    }
  }
  return bc_gemv(W, d_in, d_out, x, idx, k, y, scratch, kPartialBytes + kTicketBytes, stream);
}
