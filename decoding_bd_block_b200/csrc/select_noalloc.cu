// bd_confidence_select_noalloc: the confidence-select step for callers that
// cannot hand the library a scratch workspace.
//
// Some callers have no way to allocate device memory at the point where they
// run the step: a plugin inside a host application that only passes it
// input and output buffers, code running while a framework's caching
// allocator owns the whole device, or a latency-critical loop that must not
// hit cudaMalloc's implicit device synchronisation.  For them this file
// keeps the step's scratch (packed rows, per-row partials, counters) in one
// fixed array of device memory that belongs to the library itself.
//
// The array is a file-scope __device__ variable: every GPU on which the
// library's module is loaded holds its BD_NOALLOC_SCRATCH_BYTES until the
// process exits, whether or not this entry point is used.  Host code cannot
// pass the variable's name to a kernel (on the host it names a stand-in, not
// device memory), so its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, and cached for the life of
// the process (a cudaDeviceReset would leave the cached address stale).
//
// The scratch starts with the 16-byte header of the select workspace (the
// row count, a status word, and the arrival and tile counters of the
// single-kernel path), which the kernels expect to read as zero when a call
// starts.  Every call clears it on the caller's stream before its kernels,
// so a call that was cut short (or that overlapped another one) cannot
// leave a later, properly ordered call reading stale counters.
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "bd_common.cuh"

namespace bd {
namespace {

static __device__ __align__(256) unsigned char g_select_scratch[BD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_select_scratch on the current device (nullptr and the
// CUDA error on failure).  The first call on a device does the look-up.
void* scratch_for_current_device(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_select_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace bd

static int noalloc_call(int32_t dtype, int32_t batch, int32_t hidden, int32_t vocab,
                        const void* h, const void* h_prev, const void* w,
                        const uint32_t* masked_bits, float tau, int32_t sub_block,
                        int32_t* tokens, uint32_t* unmask_bits, float* pmax_out,
                        int32_t* argmax_out, void* stream) {
  if (batch <= 0 || batch > 65535 || hidden <= 0 || vocab <= 0) return BD_ERR_INVALID_ARG;
  if (dtype != BD_F32 && dtype != BD_BF16) return BD_ERR_UNSUPPORTED;
  // The scratch layout is the one bd_confidence_select asks its caller for;
  // a step that needs more than the fixed array is refused before anything
  // is looked up or launched.
  const bd::SelectPlan p = bd::plan_confidence_select(dtype, batch, hidden, vocab);
  if (p.total > static_cast<size_t>(BD_NOALLOC_SCRATCH_BYTES)) return BD_ERR_WORKSPACE;
  cudaError_t e = cudaSuccess;
  void* scratch = bd::scratch_for_current_device(&e);
  if (!scratch) return bd::report_cuda_error(e);  // BD_ERR_CUDA, text kept for the caller
  // the select kernels read the header as zero at the start of a call
  e = cudaMemsetAsync(scratch, 0, 16, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return bd::report_cuda_error(e);
  return bd_confidence_select(dtype, batch, hidden, vocab, h, h_prev, w, masked_bits, tau,
                              sub_block, tokens, unmask_bits, pmax_out, argmax_out, scratch,
                              static_cast<size_t>(BD_NOALLOC_SCRATCH_BYTES), stream);
}

extern "C" int bd_confidence_select_noalloc(int32_t dtype, int32_t batch, int32_t hidden,
                                            int32_t vocab, const void* h, const void* h_prev,
                                            const void* w, const uint32_t* masked_bits,
                                            float tau, int32_t sub_block, int32_t* tokens,
                                            uint32_t* unmask_bits, float* pmax_out,
                                            int32_t* argmax_out, void* stream) {
  nvtxRangePushA("bd_confidence_select_noalloc");
  const int st = noalloc_call(dtype, batch, hidden, vocab, h, h_prev, w, masked_bits, tau, sub_block,
                              tokens, unmask_bits, pmax_out, argmax_out, stream);
  nvtxRangePop();
  return st;
}

