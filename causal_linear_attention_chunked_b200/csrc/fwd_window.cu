// fwd_window.cu -- sliding-window causal linear attention.
//
// lineartile 1.0.0 ("Features") lists sliding-window attention.  For linear
// attention, row i attends to the w most recent keys, i - w < j <= i, whose
// state is the difference S_i - S_{i-w} of two prefix states:
//     O_i = phi(Q_i)(S_i - S_{i-w}) / (phi(Q_i).(z_i - z_{i-w}) + eps).
// The kernel never forms that difference of two large prefix sums (it would
// cancel as the sequence grows); per 32-token chunk c (rows c0 .. c0+31) it
// splits each row's window into three disjoint key ranges:
//   * the keys every row of the chunk sees, [max(0, c0-w+32), c0): a window
//     state [Sw | zw] carried from chunk to chunk by adding the chunk just
//     done and subtracting the keys that left (at most 32 per step), so it
//     only ever holds O(w) terms;
//   * a lag tile, [max(0, c0-w+1), the start of the range above) (fewer
//     than 32 keys), band-masked per row (j > i - w);
//   * the chunk itself, band-masked (i - w < j <= i),
// and O = (phi(Q) Sw + P_lag [V|1] + P_cur [V|1]) / (... + eps), the two-level
// structure of "Why Stream Wins at Ultra-Long Context", section 5.3 with the
// carry bounded to the window.  fp32 FMA arithmetic in shared memory, one CTA
// per (sequence, query head); bf16, fp16 or fp32 inputs and outputs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/lt_linear_attn.h"
#include "lt_internal.h"
#include "lt_ptx.cuh"

namespace lt {
namespace {

constexpr int kC = 32;   // tokens per chunk
constexpr int kT = 256;  // threads
constexpr int P = 1;     // row padding of the shared tiles (bank spread)

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
__device__ __forceinline__ void from_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void from_f(__half* p, float x) { *p = __float2half_rn(x); }
__device__ __forceinline__ float phi_w(float x) { return x > 0.0f ? x + 1.0f : expf(x); }

struct WinArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  const int32_t* cu_seqlens;
  int Hq, Hkv, N, window;
  float eps;
  int total_tokens;
  int* err;
};

// tokens [lo, hi) of head h (token-major [.][H][W]) -> rows 0 .. hi-lo-1 of
// dst [kC][W + P] (phi applied when `phi`), the other rows zero
template <typename T, int W>
__device__ __forceinline__ void load_rows(float (*dst)[W + P], const T* src, int t0, int lo,
                                          int hi, int H, int h, bool phi) {
  for (int e = threadIdx.x; e < kC * W; e += kT) {
    const int r = e / W, c = e % W;
    float x = 0.0f;
    if (lo + r < hi) {
      x = to_f(src[((size_t)(t0 + lo + r) * H + h) * W + c]);
      if (phi) x = phi_w(x);
    }
    dst[r][c] = x;
  }
}

template <int D, int DV>
struct WSmem {
  float S[D][DV + P];  // window state Sw
  float z[D];          // and zw
  float pq[kC][D + P];
  float pk[kC][D + P];  // current chunk, then the keys leaving the window
  float vv[kC][DV + P];
  float lk[kC][D + P];  // lag tile
  float lv[kC][DV + P];
  float A[kC][kC + P];  // masked scores, current chunk
  float L[kC][kC + P];  // masked scores, lag tile
  float num[kC][DV + P];
  float den[kC];
};

template <typename T, int D, int DV>
__global__ void __launch_bounds__(kT) lt_fwd_window_kernel(const WinArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  WSmem<D, DV>& sm = *reinterpret_cast<WSmem<D, DV>*>(smem_raw);
  const int tid = threadIdx.x, h = blockIdx.x, s = blockIdx.y;
  const int G = a.Hq / a.Hkv, g = h / G, w = a.window;
  int t0 = s * a.N, n = a.N;
  if (a.cu_seqlens) {
    const int lo = a.cu_seqlens[s], hi = a.cu_seqlens[s + 1];
    if (lo < 0 || hi < lo || hi > a.total_tokens) {
      if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
      return;
    }
    t0 = lo;
    n = hi - lo;
  }
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  T* out = static_cast<T*>(a.out);
  for (int i = tid; i < D * DV; i += kT) sm.S[i / DV][i % DV] = 0.0f;
  for (int i = tid; i < D; i += kT) sm.z[i] = 0.0f;
  // window state += sign * phi(K)^T [V | 1] over the rows in pk, vv
  auto add_state = [&](float sign) {
    for (int e = tid; e < D * DV; e += kT) {
      const int r = e / DV, c = e % DV;
      float x = 0.0f;
#pragma unroll 8
      for (int t = 0; t < kC; ++t) x = fmaf(sm.pk[t][r], sm.vv[t][c], x);
      sm.S[r][c] = fmaf(sign, x, sm.S[r][c]);
    }
    for (int r = tid; r < D; r += kT) {
      float x = 0.0f;
#pragma unroll 8
      for (int t = 0; t < kC; ++t) x += sm.pk[t][r];
      sm.z[r] = fmaf(sign, x, sm.z[r]);
    }
  };
  __syncthreads();
  for (int c0 = 0; c0 < n; c0 += kC) {
    const int s_lo = max(0, c0 - w + kC);               // window state: [s_lo, c0)
    const int l_lo = max(0, c0 - w + 1);                // lag tile: [l_lo, l_hi)
    const int l_hi = max(l_lo, min(c0 - w + kC, c0));
    const int c1 = min(c0 + kC, n);
    load_rows<T, D>(sm.pq, q, t0, c0, c1, a.Hq, h, true);
    load_rows<T, D>(sm.pk, k, t0, c0, c1, a.Hkv, g, true);
    load_rows<T, DV>(sm.vv, v, t0, c0, c1, a.Hkv, g, false);
    load_rows<T, D>(sm.lk, k, t0, l_lo, l_hi, a.Hkv, g, true);
    load_rows<T, DV>(sm.lv, v, t0, l_lo, l_hi, a.Hkv, g, false);
    __syncthreads();
    // band-masked scores: current chunk (i - w < j <= i), lag tile (j > i - w)
    for (int e = tid; e < 2 * kC * kC; e += kT) {
      const int lag = e >= kC * kC, r = (e % (kC * kC)) / kC, u = e % kC;
      const int i = c0 + r, j = lag ? l_lo + u : c0 + u;
      float x = 0.0f;
      if (j <= i && j > i - w && j < (lag ? l_hi : c1)) {
        const float* qr = sm.pq[r];
        const float* kr = lag ? sm.lk[u] : sm.pk[u];
#pragma unroll 8
        for (int c = 0; c < D; ++c) x = fmaf(qr[c], kr[c], x);
      }
      if (lag)
        sm.L[r][u] = x;
      else
        sm.A[r][u] = x;
    }
    __syncthreads();
    // numerator and denominator
    for (int e = tid; e < kC * DV; e += kT) {
      const int r = e / DV, c = e % DV;
      float x = 0.0f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) x = fmaf(sm.pq[r][d], sm.S[d][c], x);
#pragma unroll 8
      for (int u = 0; u < kC; ++u) x = fmaf(sm.A[r][u], sm.vv[u][c], x);
#pragma unroll 8
      for (int u = 0; u < kC; ++u) x = fmaf(sm.L[r][u], sm.lv[u][c], x);
      sm.num[r][c] = x;
    }
    for (int r = tid; r < kC; r += kT) {
      float x = a.eps;
      for (int d = 0; d < D; ++d) x = fmaf(sm.pq[r][d], sm.z[d], x);
      for (int u = 0; u < kC; ++u) x += sm.A[r][u] + sm.L[r][u];
      sm.den[r] = x;
    }
    __syncthreads();
    for (int e = tid; e < kC * DV; e += kT) {
      const int r = e / DV, c = e % DV;
      if (c0 + r < n)
        from_f(&out[((size_t)(t0 + c0 + r) * a.Hq + h) * DV + c], sm.num[r][c] / sm.den[r]);
    }
    // carry the window state to the next chunk: it becomes [s_next, c1)
    const int s_next = max(0, c0 + kC - w + kC);
    if (s_next < c1) {  // w > kC: the state is not empty
      add_state(1.0f);  // + the chunk just done (still in pk, vv)
      __syncthreads();
      if (s_lo < s_next) {  // - the keys that left: [s_lo, s_next), at most kC
        load_rows<T, D>(sm.pk, k, t0, s_lo, s_next, a.Hkv, g, true);
        load_rows<T, DV>(sm.vv, v, t0, s_lo, s_next, a.Hkv, g, false);
        __syncthreads();
        add_state(-1.0f);
      }
    }
    __syncthreads();
  }
}

template <typename T, int D, int DV>
cudaError_t launch_window_t(const WinArgs& a, int B, cudaStream_t stream) {
  const size_t smem = sizeof(WSmem<D, DV>);
  auto kern = lt_fwd_window_kernel<T, D, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.Hq, B), kT, smem, stream>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_window_w(const WinArgs& a, int B, int d, int dv, cudaStream_t stream) {
  if (d == 64 && dv == 64) return launch_window_t<T, 64, 64>(a, B, stream);
  if (d == 128 && dv == 128) return launch_window_t<T, 128, 128>(a, B, stream);
  if (d == 64 && dv == 128) return launch_window_t<T, 64, 128>(a, B, stream);
  if (d == 128 && dv == 64) return launch_window_t<T, 128, 64>(a, B, stream);
  return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace lt

extern "C" lt_status_t lt_linear_attn_fwd_window(const void* q, const void* k, const void* v,
                                                 void* out, int B, int H_q, int H_kv, int N,
                                                 int d, int dv, int window, float eps,
                                                 const int32_t* cu_seqlens, lt_stream_t stream,
                                                 lt_dtype_t dtype) {
  if (window < 1) return LT_ERR_INVALID_ARG;
  lt::FwdLaunch p;
  const lt_status_t st =
      lt::check_fwd(q, k, v, out, B, H_q, H_kv, N, d, dv, 1, eps, cu_seqlens, dtype, &p);
  if (st != LT_OK) return st;
  lt::WinArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.cu_seqlens = cu_seqlens;
  a.Hq = H_q;
  a.Hkv = H_kv;
  a.N = N;
  a.window = window;
  a.eps = eps;
  a.total_tokens = (int)p.total_tokens;
  a.err = lt::device_error_word_current();
  if (!a.err) return LT_ERR_CUDA;
  const cudaStream_t s = (cudaStream_t)stream;
  const cudaError_t e =
      dtype == LT_BF16  ? lt::launch_window_w<__nv_bfloat16>(a, B, d, dv, s)
      : dtype == LT_F16 ? lt::launch_window_w<__half>(a, B, d, dv, s)
                        : lt::launch_window_w<float>(a, B, d, dv, s);
  return e == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}
