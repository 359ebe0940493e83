// fwd_f32.cu -- chunked kernelised linear attention with fp32 I/O and fp32
// FFMA arithmetic (SIMT).
//
// Same method and chunking as the bf16 tensor-core kernel (lineartile
// 1.0.0, "How It Works"/"Reference"; chunk-local work plus an inter-chunk
// carry as in "Why Stream Wins at Ultra-Long Context", section 5.3), kept
// in fp32 end to end: tf32 or bf16 tensor-core operands would round the
// inputs to 10 or 7 mantissa bits, which cannot hold a 1e-4 relative error
// bound, so this path stays on the FMA pipes.
//
// One CTA per (sequence, query head); the CTA walks its chunks in order with
// the state [S|z] resident in shared memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lt_internal.h"
#include "lt_state.h"
#include "lt_ptx.cuh"

namespace lt {
namespace {

constexpr int kC = 32;  // tokens per chunk
constexpr int kT = 256; // threads

// the feature maps in fp32: ELU + 1 (the method's), ReLU, exp
template <int PHI>
__device__ __forceinline__ float phi_acc(float x) {
  if constexpr (PHI == kPhiElu1) return x > 0.0f ? x + 1.0f : expf(x);
  else if constexpr (PHI == kPhiRelu) return fmaxf(x, 0.0f);
  else return expf(x);
}

struct F32Args {
  const float* q;
  const float* k;
  const float* v;
  float* out;
  const int32_t* cu_seqlens;
  int Hq, Hkv, N, G, causal;
  float eps;
  int total_tokens;
  int* err;
  // optional: initial state (else zero) and final state, per (sequence, KV
  // head): S [.][Hkv][D][DV], z [.][Hkv][D]
  const float* s0;
  const float* z0;
  float* s_out;
  float* z_out;
};

template <int D, int DV, int PHI>
__global__ void __launch_bounds__(kT) lt_fwd_f32_kernel(const F32Args a) {
  extern __shared__ float sm[];
  float* S = sm;                 // D x DV
  float* z = S + D * DV;         // D
  float* pq = z + D;             // kC x D   phi(Q_c)
  float* pk = pq + kC * D;       // kC x D   phi(K_c) (zero beyond the sequence)
  float* vv = pk + kC * D;       // kC x DV
  float* P = vv + kC * DV;       // kC x kC  masked scores
  float* den = P + kC * kC;      // kC

  const int tid = threadIdx.x;
  const int h = blockIdx.x;      // query head
  const int s = blockIdx.y;      // sequence
  const int g = h / a.G;         // its KV head
  int t0, n;
  if (a.cu_seqlens) {
    const int lo = a.cu_seqlens[s], hi = a.cu_seqlens[s + 1];
    if (lo < 0 || hi < lo || hi > a.total_tokens) {
      if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
      return;
    }
    t0 = lo;
    n = hi - lo;
  } else {
    t0 = s * a.N;
    n = a.N;
  }
  const size_t sg = (size_t)s * a.Hkv + g;  // this (sequence, KV head) state
  // the CTA of the group's first query head writes the group's final state
  const bool writes_state = a.s_out != nullptr && h % a.G == 0;
  if (n <= 0) {
    if (writes_state) {
      for (int e = tid; e < D * DV; e += kT) a.s_out[sg * D * DV + e] = a.s0 ? a.s0[sg * D * DV + e] : 0.0f;
      for (int e = tid; e < D; e += kT) a.z_out[sg * D + e] = a.z0 ? a.z0[sg * D + e] : 0.0f;
    }
    return;
  }
  for (int e = tid; e < D * DV; e += kT) S[e] = a.s0 ? a.s0[sg * D * DV + e] : 0.0f;
  for (int e = tid; e < D; e += kT) z[e] = a.z0 ? a.z0[sg * D + e] : 0.0f;
  const int nc = (n + kC - 1) / kC;

  auto load_kv = [&](int c) {
    const int valid = min(kC, n - c * kC);
    for (int e = tid; e < kC * D; e += kT) {
      const int r = e / D, col = e % D;
      pk[e] = r < valid ? phi_acc<PHI>(a.k[((size_t)(t0 + c * kC + r) * a.Hkv + g) * D + col]) : 0.0f;
    }
    for (int e = tid; e < kC * DV; e += kT) {
      const int r = e / DV, col = e % DV;
      vv[e] = r < valid ? a.v[((size_t)(t0 + c * kC + r) * a.Hkv + g) * DV + col] : 0.0f;
    }
  };
  auto load_q = [&](int c) {
    const int valid = min(kC, n - c * kC);
    for (int e = tid; e < kC * D; e += kT) {
      const int r = e / D, col = e % D;
      pq[e] = r < valid ? phi_acc<PHI>(a.q[((size_t)(t0 + c * kC + r) * a.Hq + h) * D + col]) : 0.0f;
    }
  };
  // S += phi(K_c)^T V_c ; z += sum_rows phi(K_c)
  auto update_state = [&]() {
    for (int e = tid; e < D * DV; e += kT) {
      const int r = e / DV, col = e % DV;
      float acc = S[e];
      for (int t = 0; t < kC; ++t) acc = fmaf(pk[t * D + r], vv[t * DV + col], acc);
      S[e] = acc;
    }
    for (int e = tid; e < D; e += kT) {
      float acc = z[e];
      for (int t = 0; t < kC; ++t) acc += pk[t * D + e];
      z[e] = acc;
    }
  };
  // O_c = (mask(P) V_c + phi(Q_c) S) / (mask(P) 1 + phi(Q_c) z + eps)
  auto emit = [&](int c, bool intra) {
    const int valid = min(kC, n - c * kC);
    if (intra) {
      for (int e = tid; e < kC * kC; e += kT) {
        const int i = e / kC, j = e % kC;
        float acc = 0.0f;
        if (j <= i)
          for (int x = 0; x < D; ++x) acc = fmaf(pq[i * D + x], pk[j * D + x], acc);
        P[e] = acc;
      }
      __syncthreads();
    }
    for (int i = tid; i < kC; i += kT) {
      float acc = 0.0f;
      for (int x = 0; x < D; ++x) acc = fmaf(pq[i * D + x], z[x], acc);
      if (intra)
        for (int j = 0; j <= i; ++j) acc += P[i * kC + j];
      den[i] = acc + a.eps;
    }
    __syncthreads();
    for (int e = tid; e < kC * DV; e += kT) {
      const int i = e / DV, col = e % DV;
      if (i >= valid) continue;
      float acc = 0.0f;
      for (int x = 0; x < D; ++x) acc = fmaf(pq[i * D + x], S[x * DV + col], acc);
      if (intra)
        for (int j = 0; j <= i; ++j) acc = fmaf(P[i * kC + j], vv[j * DV + col], acc);
      a.out[((size_t)(t0 + c * kC + i) * a.Hq + h) * DV + col] = acc / den[i];
    }
  };

  if (a.causal) {
    for (int c = 0; c < nc; ++c) {
      load_kv(c);
      load_q(c);
      __syncthreads();
      emit(c, true);
      __syncthreads();
      update_state();
      __syncthreads();
    }
  } else {
    for (int c = 0; c < nc; ++c) {
      load_kv(c);
      __syncthreads();
      update_state();
      __syncthreads();
    }
    for (int c = 0; c < nc; ++c) {
      load_q(c);
      __syncthreads();
      emit(c, false);
      __syncthreads();
    }
  }
  if (writes_state) {  // every state update is complete (barrier above)
    for (int e = tid; e < D * DV; e += kT) a.s_out[sg * D * DV + e] = S[e];
    for (int e = tid; e < D; e += kT) a.z_out[sg * D + e] = z[e];
  }
}

template <int D, int DV, int PHI>
cudaError_t launch(const FwdLaunch& p, const float* s0, const float* z0, float* s_out,
                   float* z_out, cudaStream_t stream) {
  const int smem = (D * DV + D + 2 * kC * D + kC * DV + kC * kC + kC) * 4;
  auto kern = lt_fwd_f32_kernel<D, DV, PHI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  F32Args a;
  a.q = static_cast<const float*>(p.q);
  a.k = static_cast<const float*>(p.k);
  a.v = static_cast<const float*>(p.v);
  a.out = static_cast<float*>(p.out);
  a.cu_seqlens = p.cu_seqlens;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.N = p.N;
  a.G = p.Hq / p.Hkv;
  a.causal = p.causal;
  a.eps = p.eps;
  a.total_tokens = (int)p.total_tokens;
  a.err = p.err;
  a.s0 = s0;
  a.z0 = z0;
  a.s_out = s_out;
  a.z_out = z_out;
  kern<<<dim3(p.Hq, p.B), kT, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int PHI>
cudaError_t launch_widths(const FwdLaunch& p, const float* s0, const float* z0, float* s_out,
                          float* z_out, cudaStream_t stream) {
  if (p.d == 64 && p.dv == 64) return launch<64, 64, PHI>(p, s0, z0, s_out, z_out, stream);
  if (p.d == 128 && p.dv == 128) return launch<128, 128, PHI>(p, s0, z0, s_out, z_out, stream);
  if (p.d == 64 && p.dv == 128) return launch<64, 128, PHI>(p, s0, z0, s_out, z_out, stream);
  if (p.d == 128 && p.dv == 64) return launch<128, 64, PHI>(p, s0, z0, s_out, z_out, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_fwd_f32_state(const FwdLaunch& p, const float* s0, const float* z0,
                                 float* s_out, float* z_out, cudaStream_t stream) {
  if (p.phi == kPhiRelu) return launch_widths<kPhiRelu>(p, s0, z0, s_out, z_out, stream);
  if (p.phi == kPhiExp) return launch_widths<kPhiExp>(p, s0, z0, s_out, z_out, stream);
  return launch_widths<kPhiElu1>(p, s0, z0, s_out, z_out, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_f32(const FwdLaunch& p, cudaStream_t stream) {
  return launch_fwd_f32_state(p, nullptr, nullptr, nullptr, nullptr, stream);
}

}  // namespace lt
