// bwd.cu -- backward pass of kernelised linear attention: dQ, dK, dV for an
// upstream gradient dO of O = phi(Q) S / (phi(Q) . z + eps).
//
// lineartile 1.0.0 lists a backward pass ("Project Structure":
// core/kernels/backward.py, tests/test_backward) without a formula.  With
// a_ij = phi(Q_i).phi(K_j) over the kept pairs (j <= i causal, all j
// otherwise), den_i = sum_j a_ij + eps and O_i = sum_j a_ij V_j / den_i:
//     g_i = dO_i / den_i,   h_i = -(dO_i . O_i) / den_i,   da_ij = g_i.V_j + h_i
//     dphi(Q_i) = sum_j da_ij phi(K_j),  dphi(K_j) = sum_i da_ij phi(Q_i),
//     dV_j = sum_i a_ij g_i,   dX = dphi(X) * phi'(X),
// and phi'(x) = 1 (x > 0), e^x (x <= 0), i.e. min(phi(x), 1).  Evaluated as
// two chunked scans, each splitting the sums into the chunk itself (masked
// dense products) and the carried state, as the forward pass does ("Why
// Stream Wins at Ultra-Long Context", section 5.3; the reverse scan is the
// backward recurrence of its section 4.2):
//   1. forward scan, one CTA per (sequence, query head): the state
//      [S | z]_<c carried over chunks; per chunk O and den recomputed, G =
//      [g | h] written to a workspace, and
//          dphi(Q_c) = mask(G [V|1]^T) phi(K_c) + g S^T + h z^T;
//   2. reverse scan, one CTA per (sequence, KV head): R = sum phi(Q)^T g,
//      r = sum phi(Q)^T h over the later chunks and every query head of the
//      group, and per chunk
//          dphi(K_c) = V_c R^T + r + sum_h mask(G [V|1]^T)^T phi(Q_c),
//          dV_c      = phi(K_c) R  + sum_h mask(phi(Q) phi(K)^T)^T g.
// Non-causal: the state and R are sums over the whole sequence, computed in a
// first pass, and there are no chunk-local terms.
//
// fp32 FMA arithmetic in shared memory (bf16 or fp32 inputs and outputs,
// outputs rounded once).  The workspace holds G for every (token, query
// head): tokens * H_q * (dv + 1) floats.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/lt_linear_attn.h"
#include "lt_fault.h"
#include "lt_internal.h"
#include "lt_ptx.cuh"

namespace lt {
namespace {

constexpr int kC = 32;   // tokens per chunk
constexpr int kT = 256;  // threads

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ float phi_b(float x) { return x > 0.0f ? x + 1.0f : expf(x); }

struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  float* G;  // [tokens][Hq][dv + 1]
  const int32_t* cu_seqlens;
  int Hq, Hkv, N, causal;
  float eps;
  int total_tokens;
  int* err;
};

__device__ __forceinline__ bool seq_of(const BwdArgs& a, int s, int& t0, int& n) {
  if (a.cu_seqlens) {
    const int lo = a.cu_seqlens[s], hi = a.cu_seqlens[s + 1];
    if (lo < 0 || hi < lo || hi > a.total_tokens) return false;
    t0 = lo;
    n = hi - lo;
  } else {
    t0 = s * a.N;
    n = a.N;
  }
  return true;
}

// Row padding (floats) of the shared tiles: the products walk a tile's
// columns with the row index varying across a warp, and row strides that are
// multiples of 32 banks would put the whole warp on one bank.
constexpr int P = 1;

// rows [c0, c0 + kC) of head h of a token-major [.][H][W] tensor -> dst
// [kC][W] fp32 (phi applied when `phi`); rows past n are zero

template <typename T, int W>
__device__ __forceinline__ void load_tile(float (*dst)[W + P], const T* src, int t0, int c0, int n,
                                          int H, int h, bool phi) {
  for (int i = threadIdx.x; i < kC * W; i += kT) {
    const int r = i / W, c = i % W;
    float x = 0.0f;
    if (c0 + r < n) {
      x = to_f(src[((size_t)(t0 + c0 + r) * H + h) * W + c]);
      if (phi) x = phi_b(x);
    }
    dst[r][c] = x;
  }
}

// ---------------------------------------------------------------- kernel 1
template <typename T, int D, int DV>
struct Smem1 {
  float S[D][DV + P];
  float z[D];
  float pq[kC][D + P];
  float pk[kC][D + P];
  float vv[kC][DV + P];
  float go[kC][DV + P];  // dO, then g
  float o[kC][DV + P];   // numerator, then O
  float A[kC][kC + P];   // masked scores, then masked da
  float den[kC];
  float hh[kC];
};

template <typename T, int D, int DV>
__global__ void __launch_bounds__(kT) lt_bwd_dq_kernel(const BwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem1<T, D, DV>& sm = *reinterpret_cast<Smem1<T, D, DV>*>(smem_raw);
  const int tid = threadIdx.x, h = blockIdx.x, s = blockIdx.y;
  const int G = a.Hq / a.Hkv, g = h / G;
  int t0, n;
  if (!seq_of(a, s, t0, n)) {
    if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
    return;
  }
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const T* dout = static_cast<const T*>(a.dout);
  T* dq = static_cast<T*>(a.dq);
  for (int i = tid; i < D * DV; i += kT) sm.S[i / DV][i % DV] = 0.0f;
  for (int i = tid; i < D; i += kT) sm.z[i] = 0.0f;
  __syncthreads();
  // state update from the chunk in pk, vv
  auto advance_state = [&]() {
    for (int e = tid; e < D * DV; e += kT) {
      const int r = e / DV, c = e % DV;
      float x = sm.S[r][c];
#pragma unroll 8
      for (int t = 0; t < kC; ++t) x = fmaf(sm.pk[t][r], sm.vv[t][c], x);
      sm.S[r][c] = x;
    }
    for (int r = tid; r < D; r += kT) {
      float x = sm.z[r];
#pragma unroll 8
      for (int t = 0; t < kC; ++t) x += sm.pk[t][r];
      sm.z[r] = x;
    }
  };
  const bool causal = a.causal != 0;
  if (!causal) {  // the whole sequence's state first
    for (int c0 = 0; c0 < n; c0 += kC) {
      load_tile<T, D>(sm.pk, k, t0, c0, n, a.Hkv, g, true);
      load_tile<T, DV>(sm.vv, v, t0, c0, n, a.Hkv, g, false);
      __syncthreads();
      advance_state();
      __syncthreads();
    }
  }
  for (int c0 = 0; c0 < n; c0 += kC) {
    load_tile<T, D>(sm.pq, q, t0, c0, n, a.Hq, h, true);
    load_tile<T, D>(sm.pk, k, t0, c0, n, a.Hkv, g, true);
    load_tile<T, DV>(sm.vv, v, t0, c0, n, a.Hkv, g, false);
    load_tile<T, DV>(sm.go, dout, t0, c0, n, a.Hq, h, false);
    __syncthreads();
    if (causal) {  // masked chunk scores
      for (int e = tid; e < kC * kC; e += kT) {
        const int i = e / kC, j = e % kC;
        float x = 0.0f;
        if (j <= i) {
#pragma unroll 8
          for (int r = 0; r < D; ++r) x = fmaf(sm.pq[i][r], sm.pk[j][r], x);
        }
        sm.A[i][j] = x;
      }
      __syncthreads();
    }
    // numerator and denominator: chunk part + state part
    for (int e = tid; e < kC * DV; e += kT) {
      const int i = e / DV, c = e % DV;
      float x = 0.0f;
      if (causal) {
        for (int j = 0; j <= i; ++j) x = fmaf(sm.A[i][j], sm.vv[j][c], x);
      }
#pragma unroll 8
      for (int r = 0; r < D; ++r) x = fmaf(sm.pq[i][r], sm.S[r][c], x);
      sm.o[i][c] = x;
    }
    for (int i = tid; i < kC; i += kT) {
      float x = a.eps;
      if (causal) {
        for (int j = 0; j <= i; ++j) x += sm.A[i][j];
      }
      for (int r = 0; r < D; ++r) x = fmaf(sm.pq[i][r], sm.z[r], x);
      sm.den[i] = x;
    }
    __syncthreads();
    // O, g = dO / den, h = -(dO . O) / den; G to the workspace
    for (int i = tid; i < kC; i += kT) {
      const float inv = 1.0f / sm.den[i];
      float dot = 0.0f;
      for (int c = 0; c < DV; ++c) {
        const float oc = sm.o[i][c] * inv;
        dot = fmaf(sm.go[i][c], oc, dot);
        sm.go[i][c] *= inv;
      }
      sm.hh[i] = -dot * inv;
    }
    __syncthreads();
    for (int e = tid; e < kC * (DV + 1); e += kT) {
      const int i = e / (DV + 1), c = e % (DV + 1);
      if (c0 + i < n)
        a.G[((size_t)(t0 + c0 + i) * a.Hq + h) * (DV + 1) + c] = c < DV ? sm.go[i][c] : sm.hh[i];
    }
    if (causal) {  // masked da (overwrites the scores)
      for (int e = tid; e < kC * kC; e += kT) {
        const int i = e / kC, j = e % kC;
        float x = 0.0f;
        if (j <= i) {
          x = sm.hh[i];
#pragma unroll 8
          for (int c = 0; c < DV; ++c) x = fmaf(sm.go[i][c], sm.vv[j][c], x);
        }
        sm.A[i][j] = x;
      }
      __syncthreads();
    }
    // dphi(Q) = da phi(K) + g S^T + h z^T;  dQ = dphi(Q) * min(phi(Q), 1)
    for (int e = tid; e < kC * D; e += kT) {
      const int i = e / D, r = e % D;
      float x = sm.hh[i] * sm.z[r];
      if (causal) {
        for (int j = 0; j <= i; ++j) x = fmaf(sm.A[i][j], sm.pk[j][r], x);
      }
#pragma unroll 8
      for (int c = 0; c < DV; ++c) x = fmaf(sm.go[i][c], sm.S[r][c], x);
      if (c0 + i < n) from_f(&dq[((size_t)(t0 + c0 + i) * a.Hq + h) * D + r], x * fminf(sm.pq[i][r], 1.0f));
    }
    __syncthreads();
    if (causal) {
      advance_state();
      __syncthreads();
    }
  }
}

// ---------------------------------------------------------------- kernel 2
template <typename T, int D, int DV>
struct Smem2 {
  float R[D][DV + P];
  float r[D];
  float pk[kC][D + P];
  float vv[kC][DV + P];
  float pq[kC][D + P];
  float gg[kC][DV + P];
  float hh[kC];
  float A[kC][kC + P];
  float dA[kC][kC + P];
  float dpk[kC][D + P];
  float dvv[kC][DV + P];
};

template <typename T, int D, int DV>
__global__ void __launch_bounds__(kT) lt_bwd_dkv_kernel(const BwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem2<T, D, DV>& sm = *reinterpret_cast<Smem2<T, D, DV>*>(smem_raw);
  const int tid = threadIdx.x, g = blockIdx.x, s = blockIdx.y;
  const int G = a.Hq / a.Hkv;
  int t0, n;
  if (!seq_of(a, s, t0, n)) {
    if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
    return;
  }
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  T* dk = static_cast<T*>(a.dk);
  T* dvo = static_cast<T*>(a.dv);
  for (int i = tid; i < D * DV; i += kT) sm.R[i / DV][i % DV] = 0.0f;
  for (int i = tid; i < D; i += kT) sm.r[i] = 0.0f;
  // G rows [c0, c0 + kC) of query head h -> gg, hh (zero past n)
  auto load_g = [&](int c0, int h) {
    for (int e = tid; e < kC * (DV + 1); e += kT) {
      const int i = e / (DV + 1), c = e % (DV + 1);
      const float x = c0 + i < n ? a.G[((size_t)(t0 + c0 + i) * a.Hq + h) * (DV + 1) + c] : 0.0f;
      if (c < DV)
        sm.gg[i][c] = x;
      else
        sm.hh[i] = x;
    }
  };
  // R += phi(Q)^T g, r += phi(Q)^T h for the chunk in pq, gg, hh
  auto advance_r = [&]() {
    for (int e = tid; e < D * DV; e += kT) {
      const int rr = e / DV, c = e % DV;
      float x = sm.R[rr][c];
#pragma unroll 8
      for (int i = 0; i < kC; ++i) x = fmaf(sm.pq[i][rr], sm.gg[i][c], x);
      sm.R[rr][c] = x;
    }
    for (int rr = tid; rr < D; rr += kT) {
      float x = sm.r[rr];
#pragma unroll 8
      for (int i = 0; i < kC; ++i) x = fmaf(sm.pq[i][rr], sm.hh[i], x);
      sm.r[rr] = x;
    }
  };
  const bool causal = a.causal != 0;
  __syncthreads();
  if (!causal) {  // R, r over the whole sequence and every query head first
    for (int c0 = 0; c0 < n; c0 += kC) {
      for (int h = g * G; h < (g + 1) * G; ++h) {
        load_tile<T, D>(sm.pq, q, t0, c0, n, a.Hq, h, true);
        load_g(c0, h);
        __syncthreads();
        advance_r();
        __syncthreads();
      }
    }
  }
  const int nch = (n + kC - 1) / kC;
  for (int ci = nch - 1; ci >= 0; --ci) {
    const int c0 = ci * kC;
    load_tile<T, D>(sm.pk, k, t0, c0, n, a.Hkv, g, true);
    load_tile<T, DV>(sm.vv, v, t0, c0, n, a.Hkv, g, false);
    __syncthreads();
    // the later chunks (causal) or the whole sequence (non-causal), via R, r
    for (int e = tid; e < kC * D; e += kT) {
      const int j = e / D, rr = e % D;
      float x = sm.r[rr];
#pragma unroll 8
      for (int c = 0; c < DV; ++c) x = fmaf(sm.R[rr][c], sm.vv[j][c], x);
      sm.dpk[j][rr] = x;
    }
    for (int e = tid; e < kC * DV; e += kT) {
      const int j = e / DV, c = e % DV;
      float x = 0.0f;
#pragma unroll 8
      for (int rr = 0; rr < D; ++rr) x = fmaf(sm.R[rr][c], sm.pk[j][rr], x);
      sm.dvv[j][c] = x;
    }
    __syncthreads();
    if (causal) {
      // the chunk itself, every query head of the group; then fold the chunk into R
      for (int h = g * G; h < (g + 1) * G; ++h) {
        load_tile<T, D>(sm.pq, q, t0, c0, n, a.Hq, h, true);
        load_g(c0, h);
        __syncthreads();
        for (int e = tid; e < kC * kC; e += kT) {
          const int i = e / kC, j = e % kC;
          float x = 0.0f, y = 0.0f;
          if (j <= i) {
#pragma unroll 8
            for (int rr = 0; rr < D; ++rr) x = fmaf(sm.pq[i][rr], sm.pk[j][rr], x);
            y = sm.hh[i];
#pragma unroll 8
            for (int c = 0; c < DV; ++c) y = fmaf(sm.gg[i][c], sm.vv[j][c], y);
          }
          sm.A[i][j] = x;
          sm.dA[i][j] = y;
        }
        __syncthreads();
        for (int e = tid; e < kC * D; e += kT) {
          const int j = e / D, rr = e % D;
          float x = sm.dpk[j][rr];
          for (int i = j; i < kC; ++i) x = fmaf(sm.dA[i][j], sm.pq[i][rr], x);
          sm.dpk[j][rr] = x;
        }
        for (int e = tid; e < kC * DV; e += kT) {
          const int j = e / DV, c = e % DV;
          float x = sm.dvv[j][c];
          for (int i = j; i < kC; ++i) x = fmaf(sm.A[i][j], sm.gg[i][c], x);
          sm.dvv[j][c] = x;
        }
        advance_r();
        __syncthreads();
      }
    }
    // dK = dphi(K) * min(phi(K), 1); dV
    for (int e = tid; e < kC * D; e += kT) {
      const int j = e / D, rr = e % D;
      if (c0 + j < n)
        from_f(&dk[((size_t)(t0 + c0 + j) * a.Hkv + g) * D + rr],
               sm.dpk[j][rr] * fminf(sm.pk[j][rr], 1.0f));
    }
    for (int e = tid; e < kC * DV; e += kT) {
      const int j = e / DV, c = e % DV;
      if (c0 + j < n) from_f(&dvo[((size_t)(t0 + c0 + j) * a.Hkv + g) * DV + c], sm.dvv[j][c]);
    }
    __syncthreads();
  }
}

template <typename T, int D, int DV>
cudaError_t launch_bwd_t(const BwdArgs& a, int B, cudaStream_t stream) {
  const size_t s1 = sizeof(Smem1<T, D, DV>), s2 = sizeof(Smem2<T, D, DV>);
  auto k1 = lt_bwd_dq_kernel<T, D, DV>;
  auto k2 = lt_bwd_dkv_kernel<T, D, DV>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
  if (e != cudaSuccess) return e;
  k1<<<dim3(a.Hq, B), kT, s1, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k2<<<dim3(a.Hkv, B), kT, s2, stream>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd_w(const BwdArgs& a, int B, int d, int dv, cudaStream_t stream) {
  if (d == 64 && dv == 64) return launch_bwd_t<T, 64, 64>(a, B, stream);
  if (d == 128 && dv == 128) return launch_bwd_t<T, 128, 128>(a, B, stream);
  if (d == 64 && dv == 128) return launch_bwd_t<T, 64, 128>(a, B, stream);
  if (d == 128 && dv == 64) return launch_bwd_t<T, 128, 64>(a, B, stream);
  return cudaErrorInvalidValue;
}

bool dev_ptr(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

bool overlap(const void* x, size_t nx, const void* y, size_t ny) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(x), b = reinterpret_cast<uintptr_t>(y);
  return a < b + ny && b < a + nx;
}

}  // namespace
}  // namespace lt

extern "C" lt_status_t lt_linear_attn_bwd(const void* q, const void* k, const void* v,
                                          const void* dout, void* dq, void* dk, void* dv, int B,
                                          int H_q, int H_kv, int N, int d, int dv_w, int causal,
                                          float eps, const int32_t* cu_seqlens,
                                          lt_stream_t stream, lt_dtype_t dtype) {
  lt::FwdLaunch p;
  // q, k, v, dout and the sizes as lt_linear_attn_fwd checks them (dout in
  // the output's place)
  lt_status_t st = lt::check_fwd(q, k, v, const_cast<void*>(dout), B, H_q, H_kv, N, d, dv_w,
                                 causal, eps, cu_seqlens, dtype, &p);
  if (st != LT_OK) return st;
  if (dtype == LT_F16) return LT_ERR_UNSUPPORTED;
  if (!dq || !dk || !dv) return LT_ERR_INVALID_ARG;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(dq) | reinterpret_cast<uintptr_t>(dk) |
                        reinterpret_cast<uintptr_t>(dv);
  if (mis & 15u) return LT_ERR_INVALID_ARG;
  if (!lt::dev_ptr(dq) || !lt::dev_ptr(dk) || !lt::dev_ptr(dv)) return LT_ERR_INVALID_ARG;
  const size_t es = dtype == LT_BF16 ? 2 : 4;
  const long long T = p.total_tokens;
  const size_t nq = (size_t)T * H_q * d * es, nk = (size_t)T * H_kv * d * es;
  const size_t nv = (size_t)T * H_kv * dv_w * es, no = (size_t)T * H_q * dv_w * es;
  const void* ins[] = {q, k, v, dout};
  const size_t in_len[] = {nq, nk, nv, no};
  void* outs[] = {dq, dk, dv};
  const size_t out_len[] = {nq, nk, nv};
  for (int o = 0; o < 3; ++o) {
    for (int i = 0; i < 4; ++i)
      if (lt::overlap(outs[o], out_len[o], ins[i], in_len[i])) return LT_ERR_INVALID_ARG;
    for (int o2 = o + 1; o2 < 3; ++o2)
      if (lt::overlap(outs[o], out_len[o], outs[o2], out_len[o2])) return LT_ERR_INVALID_ARG;
  }
  int* err = lt::device_error_word_current();
  if (!err) return LT_ERR_CUDA;
  if (lt::injected_workspace_alloc_failure()) return LT_ERR_CUDA;
  const size_t gbytes = (size_t)T * H_q * (dv_w + 1) * sizeof(float);
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, gbytes, (cudaStream_t)stream) != cudaSuccess) {
    cudaGetLastError();
    return LT_ERR_CUDA;
  }
  lt::BwdArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.dout = dout;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.G = static_cast<float*>(ws);
  a.cu_seqlens = cu_seqlens;
  a.Hq = H_q;
  a.Hkv = H_kv;
  a.N = N;
  a.causal = causal;
  a.eps = eps;
  a.total_tokens = (int)T;
  a.err = err;
  cudaError_t e = dtype == LT_BF16
                      ? lt::launch_bwd_w<__nv_bfloat16>(a, B, d, dv_w, (cudaStream_t)stream)
                      : lt::launch_bwd_w<float>(a, B, d, dv_w, (cudaStream_t)stream);
  const cudaError_t f = cudaFreeAsync(ws, (cudaStream_t)stream);
  if (e == cudaSuccess) e = f;
  return e == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}
