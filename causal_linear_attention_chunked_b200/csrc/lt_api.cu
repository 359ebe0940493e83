// lt_api.cu -- the C ABI declared in include/lt_linear_attn.h: argument
// validation on the host, kernel selection, and the per-device error word.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/lt_linear_attn.h"
#include "lt_internal.h"
#include "lt_fault.h"
#include "lt_state.h"
#include "lt_ptx.cuh"

namespace {

// Kernels record asynchronous errors here (first error wins).
__device__ int g_device_error;

constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices];
int g_sm_count[kMaxDevices];
std::mutex g_err_mu;

// lt_debug_set_schedule's override (tests and ablations only)
std::atomic<int> g_sched_kernel{LT_SCHED_AUTO};
std::atomic<int> g_sched_blocks{0};

// Device address of the error word on the current device (looked up once
// per device).
int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  return g_err_ptr[dev];
}

bool is_device_ptr(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error state
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

bool width_ok(int w) { return w == 64 || w == 128; }

// The checks every forward entry point makes on its common arguments, in
// order; on LT_OK, *p describes the call.
lt_status_t check_fwd_impl(const void* q, const void* k, const void* v, void* out, int B, int H_q,
                      int H_kv, int N, int d, int dv, int causal, float eps,
                      const int32_t* cu_seqlens, lt_dtype_t dtype, lt::FwdLaunch* p) {
  if (dtype != LT_F32 && dtype != LT_BF16 && dtype != LT_F16) return LT_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out) return LT_ERR_INVALID_ARG;
  if (B <= 0 || H_q <= 0 || H_kv <= 0 || N <= 0) return LT_ERR_INVALID_ARG;
  if (H_q % H_kv != 0) return LT_ERR_INVALID_ARG;
  if (B > 65535 || H_kv > 65535) return LT_ERR_INVALID_ARG;  // grid y/z extents
  if (causal != 0 && causal != 1) return LT_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !isfinite(eps)) return LT_ERR_INVALID_ARG;
  if (!width_ok(d) || !width_ok(dv)) return LT_ERR_UNSUPPORTED;
  const long long tokens = cu_seqlens ? (long long)N : (long long)B * (long long)N;
  if (tokens >= (1ll << 31)) return LT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return LT_ERR_INVALID_ARG;
  if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return LT_ERR_INVALID_ARG;
  if (!is_device_ptr(q) || !is_device_ptr(k) || !is_device_ptr(v) || !is_device_ptr(out) ||
      (cu_seqlens && !is_device_ptr(cu_seqlens)))
    return LT_ERR_INVALID_ARG;
  const size_t es = dtype == LT_F32 ? 4 : 2;
  const size_t nq = (size_t)tokens * H_q * d * es, nk = (size_t)tokens * H_kv * d * es;
  const size_t nv = (size_t)tokens * H_kv * dv * es, no = (size_t)tokens * H_q * dv * es;
  if (overlaps(out, no, q, nq) || overlaps(out, no, k, nk) || overlaps(out, no, v, nv))
    return LT_ERR_INVALID_ARG;
  *p = lt::FwdLaunch{};
  p->in_f16 = dtype == LT_F16 ? 1 : 0;
  p->q = q;
  p->k = k;
  p->v = v;
  p->out = out;
  p->cu_seqlens = cu_seqlens;
  p->B = B;
  p->Hq = H_q;
  p->Hkv = H_kv;
  p->N = N;
  p->d = d;
  p->dv = dv;
  p->causal = causal;
  p->eps = eps;
  p->total_tokens = tokens;
  return LT_OK;
}

}  // namespace

namespace lt {
int* device_error_word_current() { return device_error_word(); }

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (g_sm_count[dev] <= 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    g_sm_count[dev] = sms;
  }
  return g_sm_count[dev];
}

int sched_kernel() { return g_sched_kernel.load(std::memory_order_relaxed); }
int sched_blocks() { return g_sched_blocks.load(std::memory_order_relaxed); }

lt_status_t check_fwd(const void* q, const void* k, const void* v, void* out, int B, int H_q,
                      int H_kv, int N, int d, int dv, int causal, float eps,
                      const int32_t* cu_seqlens, lt_dtype_t dtype, FwdLaunch* p) {
  return check_fwd_impl(q, k, v, out, B, H_q, H_kv, N, d, dv, causal, eps, cu_seqlens, dtype, p);
}
}  // namespace lt

extern "C" {

int lt_abi_version(void) { return 1; }

const char* lt_status_string(lt_status_t s) {
  switch (s) {
    case LT_OK: return "LT_OK";
    case LT_ERR_INVALID_ARG: return "LT_ERR_INVALID_ARG: invalid argument";
    case LT_ERR_UNSUPPORTED: return "LT_ERR_UNSUPPORTED: unsupported width or dtype";
    case LT_ERR_CUDA: return "LT_ERR_CUDA: CUDA runtime or launch failure";
    case LT_ERR_DEVICE_TIMEOUT: return "LT_ERR_DEVICE_TIMEOUT: a kernel gave up a stalled wait";
    case LT_ERR_DEVICE_BAD_SEQLENS: return "LT_ERR_DEVICE_BAD_SEQLENS: inconsistent cu_seqlens";
    case LT_ERR_SCRATCH_TOO_SMALL:
      return "LT_ERR_SCRATCH_TOO_SMALL: the shape needs more than the fixed scratch array holds";
  }
  return "unknown lt_status_t";
}

lt_status_t lt_linear_attn_fwd(const void* q, const void* k, const void* v, void* out, int B,
                               int H_q, int H_kv, int N, int d, int dv, int causal, float eps,
                               const int32_t* cu_seqlens, lt_stream_t stream,
                               lt_dtype_t dtype) {
  return lt_linear_attn_fwd_ex(q, k, v, out, B, H_q, H_kv, N, d, dv, causal, eps, cu_seqlens,
                               stream, dtype, LT_PHI_ELU1);
}

lt_status_t lt_linear_attn_fwd_ex(const void* q, const void* k, const void* v, void* out, int B,
                                  int H_q, int H_kv, int N, int d, int dv, int causal, float eps,
                                  const int32_t* cu_seqlens, lt_stream_t stream,
                                  lt_dtype_t dtype, lt_feature_map_t phi) {
  // the feature map, and the widths of the tensor-core path's variants
  // (fp16 I/O, the other maps): d = dv = 64 or 128
  if (phi != LT_PHI_ELU1 && phi != LT_PHI_RELU && phi != LT_PHI_EXP) return LT_ERR_INVALID_ARG;
  if ((dtype == LT_F16 || (dtype == LT_BF16 && phi != LT_PHI_ELU1)) &&
      !(d == dv && (d == 64 || d == 128)))
    return LT_ERR_UNSUPPORTED;
  lt::FwdLaunch p;
  const lt_status_t st =
      check_fwd_impl(q, k, v, out, B, H_q, H_kv, N, d, dv, causal, eps, cu_seqlens, dtype, &p);
  if (st != LT_OK) return st;
  p.phi = (int)phi;
  p.err = device_error_word();
  if (!p.err) return LT_ERR_CUDA;
  const cudaError_t e = dtype == LT_F32 ? lt::launch_fwd_f32(p, (cudaStream_t)stream)
                                        : lt::launch_fwd_bf16(p, (cudaStream_t)stream);
  return e == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status_t lt_linear_attn_fwd_plan(int B, int H_q, int H_kv, int N, int d, int dv, int causal,
                                    int packed, lt_dtype_t dtype, int num_sms, int* blocks,
                                    int* launches, size_t* workspace_bytes) {
  if (dtype != LT_F32 && dtype != LT_BF16 && dtype != LT_F16) return LT_ERR_UNSUPPORTED;
  if (!blocks || !launches || !workspace_bytes) return LT_ERR_INVALID_ARG;
  if (B <= 0 || H_q <= 0 || H_kv <= 0 || N <= 0 || H_q % H_kv != 0) return LT_ERR_INVALID_ARG;
  if (B > 65535 || H_kv > 65535) return LT_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return LT_ERR_INVALID_ARG;
  if (packed != 0 && packed != 1) return LT_ERR_INVALID_ARG;
  if (!width_ok(d) || !width_ok(dv)) return LT_ERR_UNSUPPORTED;
  const long long tokens = packed ? (long long)N : (long long)B * (long long)N;
  if (tokens >= (1ll << 31)) return LT_ERR_INVALID_ARG;
  if (dtype == LT_F32) {
    *blocks = 1;
    *launches = 1;
    *workspace_bytes = 0;
    return LT_OK;
  }
  if (num_sms <= 0) {
    num_sms = lt::device_sm_count();
    if (num_sms <= 0) return LT_ERR_CUDA;
  }
  lt::FwdLaunch p = {};
  p.cu_seqlens = packed ? reinterpret_cast<const int32_t*>(16) : nullptr;  // only tested for null
  p.B = B;
  p.Hq = H_q;
  p.Hkv = H_kv;
  p.N = N;
  p.d = d;
  p.dv = dv;
  p.causal = causal;
  p.total_tokens = tokens;
  p.in_f16 = dtype == LT_F16 ? 1 : 0;
  if (p.in_f16 && !(d == dv && (d == 64 || d == 128))) return LT_ERR_UNSUPPORTED;
  lt::plan_fwd_bf16(p, num_sms, blocks, launches, workspace_bytes);
  return LT_OK;
}

lt_status_t lt_linear_attn_fwd_state(const void* q, const void* k, const void* v, void* out,
                                     int B, int H_q, int H_kv, int N, int d, int dv, int causal,
                                     float eps, const int32_t* cu_seqlens, const float* S0,
                                     const float* z0, float* S_out, float* z_out,
                                     lt_stream_t stream, lt_dtype_t dtype) {
  lt::FwdLaunch p;
  const lt_status_t st =
      check_fwd_impl(q, k, v, out, B, H_q, H_kv, N, d, dv, causal, eps, cu_seqlens, dtype, &p);
  if (st != LT_OK) return st;
  if (dtype == LT_F16) return LT_ERR_UNSUPPORTED;
  if ((S0 == nullptr) != (z0 == nullptr) || (S_out == nullptr) != (z_out == nullptr))
    return LT_ERR_INVALID_ARG;
  if ((S0 && (!aligned16(S0) || (reinterpret_cast<uintptr_t>(z0) & 3u))) ||
      (S_out && (!aligned16(S_out) || (reinterpret_cast<uintptr_t>(z_out) & 3u))))
    return LT_ERR_INVALID_ARG;
  if ((S0 && (!is_device_ptr(S0) || !is_device_ptr(z0))) ||
      (S_out && (!is_device_ptr(S_out) || !is_device_ptr(z_out))))
    return LT_ERR_INVALID_ARG;
  const long long tokens = p.total_tokens;
  const size_t es = dtype == LT_BF16 ? 2 : 4;
  const size_t nq = (size_t)tokens * H_q * d * es, nk = (size_t)tokens * H_kv * d * es;
  const size_t nv = (size_t)tokens * H_kv * dv * es, no = (size_t)tokens * H_q * dv * es;
  const size_t ns = (size_t)B * H_kv * d * dv * 4, nz = (size_t)B * H_kv * d * 4;
  if (S0 && (overlaps(out, no, S0, ns) || overlaps(out, no, z0, nz))) return LT_ERR_INVALID_ARG;
  if (S_out) {
    // the final state is written while inputs may still be read: no overlap
    const void* ins[] = {q, k, v, out, S0, z0};
    const size_t lens[] = {nq, nk, nv, no, S0 ? ns : 0, S0 ? nz : 0};
    for (int i = 0; i < 6; ++i)
      if (ins[i] && (overlaps(S_out, ns, ins[i], lens[i]) || overlaps(z_out, nz, ins[i], lens[i])))
        return LT_ERR_INVALID_ARG;
    if (overlaps(S_out, ns, z_out, nz)) return LT_ERR_INVALID_ARG;
  }
  p.err = device_error_word();
  if (!p.err) return LT_ERR_CUDA;
  const cudaError_t e =
      lt::launch_fwd_state(p, dtype == LT_BF16, S0, z0, S_out, z_out, (cudaStream_t)stream);
  return e == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status_t lt_debug_set_schedule(lt_schedule_t kernel, int blocks) {
  if (kernel != LT_SCHED_AUTO && kernel != LT_SCHED_TWO_LAUNCH && kernel != LT_SCHED_GENERAL)
    return LT_ERR_INVALID_ARG;
  if (blocks < 0) return LT_ERR_INVALID_ARG;
  g_sched_kernel.store((int)kernel, std::memory_order_relaxed);
  g_sched_blocks.store(blocks, std::memory_order_relaxed);
  return LT_OK;
}

lt_status_t lt_selftest_wait_timeout(unsigned int limit_us, lt_stream_t stream) {
  if (limit_us == 0 || limit_us > 1000000u) return LT_ERR_INVALID_ARG;
  int* err = device_error_word();
  if (!err) return LT_ERR_CUDA;
  const cudaError_t e =
      lt::launch_selftest_wait(err, (uint64_t)limit_us * 1000u, (cudaStream_t)stream);
  return e == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status_t lt_linear_attn_decode_step(const void* q, const void* k, const void* v, float* S,
                                       float* z, void* out, int B, int H_q, int H_kv, int d,
                                       int dv, float eps, lt_stream_t stream,
                                       lt_dtype_t dtype) {
  if (dtype != LT_F32 && dtype != LT_BF16) return LT_ERR_UNSUPPORTED;
  if (!q || !k || !v || !S || !z || !out) return LT_ERR_INVALID_ARG;
  if (B <= 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0) return LT_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !isfinite(eps)) return LT_ERR_INVALID_ARG;
  if (!width_ok(d) || !width_ok(dv)) return LT_ERR_UNSUPPORTED;
  if (B > 65535) return LT_ERR_INVALID_ARG;
  if (!aligned16(S) || (reinterpret_cast<uintptr_t>(z) & 3u)) return LT_ERR_INVALID_ARG;
  if (!is_device_ptr(q) || !is_device_ptr(k) || !is_device_ptr(v) || !is_device_ptr(S) ||
      !is_device_ptr(z) || !is_device_ptr(out))
    return LT_ERR_INVALID_ARG;
  const size_t es = dtype == LT_BF16 ? 2 : 4;
  const size_t no = (size_t)B * H_q * dv * es;
  if (overlaps(out, no, q, (size_t)B * H_q * d * es) ||
      overlaps(out, no, k, (size_t)B * H_kv * d * es) ||
      overlaps(out, no, v, (size_t)B * H_kv * dv * es) ||
      overlaps(out, no, S, (size_t)B * H_kv * d * dv * 4) ||
      overlaps(out, no, z, (size_t)B * H_kv * d * 4) ||
      overlaps(S, (size_t)B * H_kv * d * dv * 4, z, (size_t)B * H_kv * d * 4))
    return LT_ERR_INVALID_ARG;
  lt::DecodeLaunch p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.S = S;
  p.z = z;
  p.out = out;
  p.B = B;
  p.Hq = H_q;
  p.Hkv = H_kv;
  p.d = d;
  p.dv = dv;
  p.eps = eps;
  p.bf16 = dtype == LT_BF16;
  return lt::launch_decode(p, (cudaStream_t)stream) == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status_t lt_get_last_device_error(lt_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return LT_ERR_CUDA;
  int* err = device_error_word();
  if (!err) return LT_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LT_ERR_CUDA;
  if (code != 0) {
    const int zero = 0;
    if (cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return LT_ERR_CUDA;
  }
  if (code == lt::kDevErrTimeout) return LT_ERR_DEVICE_TIMEOUT;
  if (code == lt::kDevErrBadSeqlens) return LT_ERR_DEVICE_BAD_SEQLENS;
  return code == 0 ? LT_OK : LT_ERR_CUDA;
}

}  // extern "C"
