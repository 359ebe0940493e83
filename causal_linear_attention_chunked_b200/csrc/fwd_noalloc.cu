// fwd_noalloc.cu -- lt_linear_attn_fwd_noalloc: the bf16 forward pass with
// the per-block partial states kept in a fixed device array that the library
// owns, so that a call allocates no memory at all.
//
// lt_linear_attn_fwd cuts each dense sequence into blocks and takes a
// stream-ordered workspace (cudaMallocAsync) for the blocks' partial states.
// Some callers cannot let a library allocate: a program whose device memory
// is all handed to its own caching allocator at start-up (a stream-ordered
// allocation from the default pool may then fail although the program has
// memory to spare), a device or driver set-up without stream-ordered
// allocation (memory pools unsupported), or code that must have a fixed
// memory footprint and no allocator work in its launch path.  This entry
// point runs the same kernels with the workspace taken from g_scratch below.
//
// Sharing: every call on a device uses the same array.  Two calls whose work
// can overlap on the GPU (different streams without an ordering between
// them, or different host threads) race on it and may return wrong results;
// order such calls.  The array keeps the previous call's contents; nothing in
// it has to start at zero, because the state launch writes every partial
// state (zeros for a block past the end of its sequence) before the forward
// launch of the same call reads it.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/lt_linear_attn.h"
#include "lt_internal.h"

namespace {

constexpr size_t kScratchBytes = LT_NOALLOC_SCRATCH_BYTES;

// Block partial states, fp32.  Every device that loads the library holds it
// until the process exits.  Host code must not pass g_scratch itself to a
// kernel: on the host the name refers to a host-side shadow object, not to
// device memory; the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) float g_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
float* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_scratch on the current device, looked up on the first
// call per device (with that device current) and cached.
cudaError_t scratch_address(float** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  *addr = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

lt_status_t lt_linear_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                       int B, int H_q, int H_kv, int N, int d, int dv,
                                       int causal, float eps, const int32_t* cu_seqlens,
                                       lt_stream_t stream) {
  // the checks of lt_linear_attn_fwd, in the same order (so the same bad
  // arguments give the same status), then the block count and workspace
  // size that call would use on this device
  lt::FwdLaunch p;
  lt_status_t st = lt::check_fwd(q, k, v, out, B, H_q, H_kv, N, d, dv, causal, eps, cu_seqlens,
                                 LT_BF16, &p);
  if (st != LT_OK) return st;
  int nb = 1, launches = 1;
  size_t ws_bytes = 0;
  st = lt_linear_attn_fwd_plan(B, H_q, H_kv, N, d, dv, causal, cu_seqlens ? 1 : 0, LT_BF16, 0,
                               &nb, &launches, &ws_bytes);
  if (st != LT_OK) return st;
  if (ws_bytes > kScratchBytes) return LT_ERR_SCRATCH_TOO_SMALL;
  p.err = lt::device_error_word_current();
  if (!p.err) return LT_ERR_CUDA;
  float* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) {
    cudaGetLastError();
    return LT_ERR_CUDA;
  }
  const cudaError_t e =
      lt::launch_fwd_bf16_ws(p, nb, ws_bytes ? scratch : nullptr, (cudaStream_t)stream);
  return e == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

}  // extern "C"
