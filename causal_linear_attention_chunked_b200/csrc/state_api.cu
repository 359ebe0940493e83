// state_api.cu -- the state without the outputs, and the carry of a sequence
// cut into segments (context parallelism).
//
// For linear attention the whole past of a sequence is the fixed-size state
// (lineartile 1.0.0, "Reference": the recurrent view of the cited linear
// attention; "Features": KV-cache reuse and multi-GPU sharding), and a
// sequence cut into contiguous segments splits exactly along it: segment r
// starts from the sum of the states of the segments before it, the carry of
// the two-level scan of "Why Stream Wins at Ultra-Long Context", section
// 5.3, taken across devices instead of across blocks.
//
//   lt_linear_attn_state        S = S0 + sum_t phi(K_t)^T V_t, z = z0 + sum_t phi(K_t)
//                               per (sequence, KV head), no outputs, no Q.
//   lt_linear_attn_state_carry  from every segment's state (gathered from the
//                               ranks), segment `rank`'s starting state: the
//                               sum over the earlier segments (causal) or the
//                               other segments (non-causal), in rank order.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/lt_linear_attn.h"
#include "lt_fault.h"
#include "lt_internal.h"
#include "lt_ptx.cuh"
#include "lt_state.h"

namespace lt {
namespace {

constexpr int kT = 256;  // threads
constexpr int kC = 32;   // tokens per tile (fp32 path)

__device__ __forceinline__ float phi_f32(float x) { return x > 0.0f ? x + 1.0f : expf(x); }

// fp32 inputs: one CTA per (KV head, sequence) walks the tokens in tiles of
// kC; thread t owns the state entries t, t + kT, ... of S (row-major d x dv)
// and, for t < d, z[t].  fp32 FMA arithmetic throughout.
template <int D, int DV>
__global__ void __launch_bounds__(kT)
    lt_state_f32_kernel(const float* __restrict__ k, const float* __restrict__ v,
                        const int32_t* cu_seqlens, int Hkv, int N, int total_tokens,
                        const float* s0, const float* z0, float* s_out, float* z_out, int* err) {
  __shared__ float pk[kC][D];
  __shared__ float vv[kC][DV];
  constexpr int PER = D * DV / kT;
  const int tid = threadIdx.x, g = blockIdx.x, s = blockIdx.y;
  int t0 = s * N, n = N;
  if (cu_seqlens) {
    const int lo = cu_seqlens[s], hi = cu_seqlens[s + 1];
    if (lo < 0 || hi < lo || hi > total_tokens) {
      if (tid == 0) report_error(err, kDevErrBadSeqlens);
      return;
    }
    t0 = lo;
    n = hi - lo;
  }
  const size_t lane = (size_t)s * Hkv + g;
  float acc[PER];
  float zacc = 0.0f;
#pragma unroll
  for (int m = 0; m < PER; ++m) acc[m] = s0 ? s0[lane * D * DV + tid + m * kT] : 0.0f;
  if (tid < D && z0) zacc = z0[lane * D + tid];
  for (int c0 = 0; c0 < n; c0 += kC) {
    for (int i = tid; i < kC * D; i += kT) {
      const int t = i / D, a = i % D;
      pk[t][a] = c0 + t < n ? phi_f32(k[((size_t)(t0 + c0 + t) * Hkv + g) * D + a]) : 0.0f;
    }
    for (int i = tid; i < kC * DV; i += kT) {
      const int t = i / DV, c = i % DV;
      vv[t][c] = c0 + t < n ? v[((size_t)(t0 + c0 + t) * Hkv + g) * DV + c] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < PER; ++m) {
      const int e = tid + m * kT, a = e / DV, c = e % DV;
      float x = acc[m];
#pragma unroll 8
      for (int t = 0; t < kC; ++t) x = fmaf(pk[t][a], vv[t][c], x);
      acc[m] = x;
    }
    if (tid < D) {
#pragma unroll 8
      for (int t = 0; t < kC; ++t) zacc += pk[t][tid];
    }
    __syncthreads();
  }
#pragma unroll
  for (int m = 0; m < PER; ++m) s_out[lane * D * DV + tid + m * kT] = acc[m];
  if (tid < D) z_out[lane * D + tid] = zacc;
}

template <int D, int DV>
cudaError_t launch_state_f32(const FwdLaunch& p, const float* s0, const float* z0, float* s_out,
                             float* z_out, cudaStream_t stream) {
  lt_state_f32_kernel<D, DV><<<dim3(p.Hkv, p.B), kT, 0, stream>>>(
      static_cast<const float*>(p.k), static_cast<const float*>(p.v), p.cu_seqlens, p.Hkv, p.N,
      (int)p.total_tokens, s0, z0, s_out, z_out, p.err);
  return cudaGetLastError();
}

// out[i] = sum over the selected segments r (in rank order) of all[r][i]:
// r < rank (causal) or r != rank (non-causal).
__global__ void __launch_bounds__(kT)
    lt_state_carry_kernel(const float* __restrict__ s_all, const float* __restrict__ z_all,
                          long long ns, long long nz, int world, int rank, int causal,
                          float* s_out, float* z_out) {
  const long long stride = (long long)gridDim.x * kT;
  for (long long i = (long long)blockIdx.x * kT + threadIdx.x; i < ns + nz; i += stride) {
    const bool in_s = i < ns;
    const float* src = in_s ? s_all + i : z_all + (i - ns);
    const long long step = in_s ? ns : nz;
    float acc = 0.0f;
    for (int r = 0; r < world; ++r)
      if (causal ? r < rank : r != rank) acc += src[(long long)r * step];
    if (in_s)
      s_out[i] = acc;
    else
      z_out[i - ns] = acc;
  }
}

bool aligned(const void* p, unsigned int a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool on_device(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

bool width_ok(int w) { return w == 64 || w == 128; }

}  // namespace

cudaError_t launch_state_only(const FwdLaunch& p, bool bf16, const float* s0, const float* z0,
                              float* s_out, float* z_out, cudaStream_t stream) {
  if (!bf16) {
    if (p.d == 64 && p.dv == 64) return launch_state_f32<64, 64>(p, s0, z0, s_out, z_out, stream);
    if (p.d == 128 && p.dv == 128)
      return launch_state_f32<128, 128>(p, s0, z0, s_out, z_out, stream);
    if (p.d == 64 && p.dv == 128) return launch_state_f32<64, 128>(p, s0, z0, s_out, z_out, stream);
    if (p.d == 128 && p.dv == 64) return launch_state_f32<128, 64>(p, s0, z0, s_out, z_out, stream);
    return cudaErrorInvalidValue;
  }
  // bf16: every block's aggregate on the tensor cores (the state launch in
  // its all-blocks mode), then the blocks summed in order onto S0
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int nb = block_count(p, sms);
  const size_t E = (size_t)p.d * p.dv + p.d;
  const size_t bytes = (size_t)p.B * p.Hkv * nb * E * sizeof(float);
  if (injected_workspace_alloc_failure()) return cudaErrorMemoryAllocation;
  void* ws = nullptr;
  cudaError_t e = cudaMallocAsync(&ws, bytes, stream);
  if (e != cudaSuccess) return e;
  FwdLaunch all = p;
  all.causal = 0;
  e = launch_block_state(all, nb, static_cast<float*>(ws), stream);
  if (e == cudaSuccess)
    e = launch_state_prefix(all, nb, static_cast<float*>(ws), s0, z0, s_out, z_out, stream);
  const cudaError_t f = cudaFreeAsync(ws, stream);
  return e != cudaSuccess ? e : f;
}

}  // namespace lt

using lt::aligned;
using lt::on_device;
using lt::overlap;
using lt::width_ok;

extern "C" {

lt_status_t lt_linear_attn_state(const void* k, const void* v, int B, int H_kv, int N, int d,
                                 int dv, const int32_t* cu_seqlens, const float* S0,
                                 const float* z0, float* S_out, float* z_out, lt_stream_t stream,
                                 lt_dtype_t dtype) {
  if (dtype != LT_F32 && dtype != LT_BF16) return LT_ERR_UNSUPPORTED;
  if (!k || !v || !S_out || !z_out) return LT_ERR_INVALID_ARG;
  if ((S0 == nullptr) != (z0 == nullptr)) return LT_ERR_INVALID_ARG;
  if (B <= 0 || H_kv <= 0 || N <= 0 || B > 65535 || H_kv > 65535) return LT_ERR_INVALID_ARG;
  if (!width_ok(d) || !width_ok(dv)) return LT_ERR_UNSUPPORTED;
  const long long tokens = cu_seqlens ? (long long)N : (long long)B * (long long)N;
  if (tokens >= (1ll << 31)) return LT_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(S_out, 16) || !aligned(z_out, 4) ||
      (S0 && (!aligned(S0, 16) || !aligned(z0, 4))) || (cu_seqlens && !aligned(cu_seqlens, 4)))
    return LT_ERR_INVALID_ARG;
  if (!on_device(k) || !on_device(v) || !on_device(S_out) || !on_device(z_out) ||
      (S0 && (!on_device(S0) || !on_device(z0))) || (cu_seqlens && !on_device(cu_seqlens)))
    return LT_ERR_INVALID_ARG;
  const size_t es = dtype == LT_BF16 ? 2 : 4;
  const size_t nk = (size_t)tokens * H_kv * d * es, nv = (size_t)tokens * H_kv * dv * es;
  const size_t ns = (size_t)B * H_kv * d * dv * 4, nz = (size_t)B * H_kv * d * 4;
  const void* ins[] = {k, v, S0, z0};
  const size_t lens[] = {nk, nv, ns, nz};
  for (int i = 0; i < 4; ++i)
    if (overlap(S_out, ns, ins[i], lens[i]) || overlap(z_out, nz, ins[i], lens[i]))
      return LT_ERR_INVALID_ARG;
  if (overlap(S_out, ns, z_out, nz)) return LT_ERR_INVALID_ARG;
  lt::FwdLaunch p = {};
  p.q = k;  // unused: the state reads only K and V
  p.k = k;
  p.v = v;
  p.cu_seqlens = cu_seqlens;
  p.B = B;
  p.Hq = H_kv;
  p.Hkv = H_kv;
  p.N = N;
  p.d = d;
  p.dv = dv;
  p.causal = 0;
  p.total_tokens = tokens;
  p.err = lt::device_error_word_current();
  if (!p.err) return LT_ERR_CUDA;
  const cudaError_t e =
      lt::launch_state_only(p, dtype == LT_BF16, S0, z0, S_out, z_out, (cudaStream_t)stream);
  return e == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

lt_status_t lt_linear_attn_state_carry(const float* S_all, const float* z_all, int world,
                                       int rank, int causal, int B, int H_kv, int d, int dv,
                                       float* S_out, float* z_out, lt_stream_t stream) {
  if (!S_all || !z_all || !S_out || !z_out) return LT_ERR_INVALID_ARG;
  if (world <= 0 || rank < 0 || rank >= world) return LT_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return LT_ERR_INVALID_ARG;
  if (B <= 0 || H_kv <= 0 || d <= 0 || dv <= 0) return LT_ERR_INVALID_ARG;
  if (!width_ok(d) || !width_ok(dv)) return LT_ERR_UNSUPPORTED;
  if (!aligned(S_all, 4) || !aligned(z_all, 4) || !aligned(S_out, 4) || !aligned(z_out, 4))
    return LT_ERR_INVALID_ARG;
  if (!on_device(S_all) || !on_device(z_all) || !on_device(S_out) || !on_device(z_out))
    return LT_ERR_INVALID_ARG;
  const long long ns = (long long)B * H_kv * d * dv, nz = (long long)B * H_kv * d;
  const size_t bs = (size_t)ns * 4, bz = (size_t)nz * 4;
  if (overlap(S_out, bs, S_all, bs * world) || overlap(S_out, bs, z_all, bz * world) ||
      overlap(z_out, bz, S_all, bs * world) || overlap(z_out, bz, z_all, bz * world) ||
      overlap(S_out, bs, z_out, bz))
    return LT_ERR_INVALID_ARG;
  const int sms = lt::device_sm_count();
  if (sms <= 0) return LT_ERR_CUDA;
  const long long blocks = (ns + nz + lt::kT - 1) / lt::kT;
  const int grid = (int)(blocks < 4LL * sms ? blocks : 4LL * sms);
  lt::lt_state_carry_kernel<<<grid, lt::kT, 0, (cudaStream_t)stream>>>(S_all, z_all, ns, nz,
                                                                       world, rank, causal,
                                                                       S_out, z_out);
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}

}  // extern "C"
