// qlora_linear_fwd_noalloc: the forward linear for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs
// where cudaMalloc is forbidden or unavailable (a custom allocator's own hooks,
// a real-time or embedded runtime that fixes its memory map at start-up, or a
// plugin host that owns every allocation).  This entry point takes only the
// inputs and outputs and runs the ordinary forward with its scratch taken from
// one array that lives in the library itself.  It launches kernels, so like
// any CUDA call it cannot be made from a stream host callback.
//
// The array is a file-scope __device__ variable of kStaticScratchBytes bytes:
// every GPU on which the library's device code is loaded holds it until the
// process exits.  Host code cannot use the array's name as a device address
// (on the host it names a shadow object), so the device address is looked up
// with cudaGetSymbolAddress once per device, with that device current, on the
// first call made on that device.  That first call should therefore come
// before any stream capture.  All calls share the array and it keeps the
// previous call's contents; the forward overwrites every scratch element it
// reads, so nothing needs clearing.  Calls that overlap on the GPU (two
// streams, or two host threads) race on the array.  The address is cached for
// the life of the process, so the device must not be reset after the first
// call (a reset reloads the module, and the array may move).
//
// The array covers the forward's minimum workspace only: the minimum grows
// with M r (about 2.4 KB per token at r = 64, so M <= 3413 there), and the
// fused GEMM's optional stream-K region (about 80 MB for M > 128) never fits,
// so the GEMM always runs without the stream-K split of a partial last wave.
#include <mutex>

#include "internal.h"

namespace qlora {
namespace {

constexpr size_t kStaticScratchBytes = QLORA_STATIC_SCRATCH_BYTES;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device (nullptr on error).
void *static_scratch_ptr() {
  static void *ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

}  // namespace
}  // namespace qlora

extern "C" qlora_status qlora_linear_fwd_noalloc(const qlora_nf4_weight *w, const uint16_t *X, int64_t M,
                                                 const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *Y,
                                                 float *H_out, void *stream) {
  if (!w) return QLORA_ERR_INVALID_ARG;
  const size_t need = qlora_workspace_min_bytes(QLORA_OP_FWD, M, w->rows, w->cols, r);
  if (need > qlora::kStaticScratchBytes) return QLORA_ERR_WORKSPACE;   // sizes beyond the static scratch
  void *scratch = qlora::static_scratch_ptr();
  if (!scratch) return QLORA_ERR_CUDA;
  return qlora_linear_fwd(w, X, M, A, B, r, s, Y, H_out, scratch, qlora::kStaticScratchBytes, stream);
}
