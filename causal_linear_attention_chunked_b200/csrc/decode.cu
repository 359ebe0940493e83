// decode.cu -- one recurrent decode step over the fixed-size state.
//
// For linear attention the KV cache of the lineartile page's "KV Cache
// Reuse" / "Flash Decoding" features is the per-head state (S, z) of the
// recurrent view (lineartile 1.0.0, "Reference": Katharopoulos et al.
// 2020; "Why Stream Wins at Ultra-Long Context", section 3.2: a fixed-size
// state per layer instead of a growing cache).  One step, per batch row b
// and KV head g, updating before reading so token i sees j <= i:
//     S += phi(k)^T v,   z += phi(k)
//     out_h = phi(q_h) S / (phi(q_h) . z + eps)   for each query head h of g.
//
// Bandwidth-bound: S (fp32, d x dv) is read and written once per step with
// 128-bit accesses; the G query heads of the group reuse the updated rows
// from registers.  One CTA per (b, g); each thread owns four consecutive
// columns of RPT rows; column sums are reduced with warp shuffles and then
// across warps through shared memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lt_internal.h"
#include "lt_ptx.cuh"

namespace lt {
namespace {

constexpr int kT = 256;

template <bool BF16>
__device__ __forceinline__ float ld_in(const void* p, size_t i) {
  if (BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  return static_cast<const float*>(p)[i];
}

__device__ __forceinline__ float phi_dec(float x) { return x > 0.0f ? x + 1.0f : expf(x); }

template <int D, int DV, bool BF16>
__global__ void __launch_bounds__(kT) lt_decode_kernel(const DecodeLaunch a) {
  constexpr int CG = DV / 4;       // column groups (float4 each)
  constexpr int RG = kT / CG;      // row groups
  constexpr int RPT = D / RG;      // rows per thread
  constexpr int NW = kT / 32;
  static_assert(RPT >= 1 && D % RG == 0, "shape");
  __shared__ float s_pk[D];
  __shared__ float s_v[DV];
  __shared__ float s_red[NW][DV];
  __shared__ float s_den[NW];
  extern __shared__ float s_pq[];  // G x D

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.x, b = blockIdx.y;
  const int G = a.Hq / a.Hkv;
  const int cg = tid % CG, rg = tid / CG;
  const size_t kv = (size_t)b * a.Hkv + g;
  float* S = a.S + kv * D * DV;
  float* z = a.z + kv * D;
  // this thread's state rows first: their loads are in flight while q, k, v
  // are staged
  float4 rows[RPT];
  float zr[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int row = rg * RPT + r;
    rows[r] = *reinterpret_cast<const float4*>(S + (size_t)row * DV + cg * 4);
    zr[r] = cg == 0 ? z[row] : 0.0f;
  }

  for (int e = tid; e < D; e += kT) s_pk[e] = phi_dec(ld_in<BF16>(a.k, kv * D + e));
  for (int e = tid; e < DV; e += kT) s_v[e] = ld_in<BF16>(a.v, kv * DV + e);
  for (int e = tid; e < G * D; e += kT)
    s_pq[e] = phi_dec(ld_in<BF16>(a.q, ((size_t)b * a.Hq + (size_t)g * G) * D + e));
  __syncthreads();

  const float4 v4 = *reinterpret_cast<const float4*>(&s_v[cg * 4]);
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int row = rg * RPT + r;
    float4 x = rows[r];
    const float pk = s_pk[row];
    x.x = fmaf(pk, v4.x, x.x);
    x.y = fmaf(pk, v4.y, x.y);
    x.z = fmaf(pk, v4.z, x.z);
    x.w = fmaf(pk, v4.w, x.w);
    *reinterpret_cast<float4*>(S + (size_t)row * DV + cg * 4) = x;
    rows[r] = x;
    if (cg == 0) {
      zr[r] += pk;
      z[row] = zr[r];
    }
  }

  for (int h = 0; h < G; ++h) {
    const float* pq = s_pq + h * D;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float dacc = 0.0f;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const float w = pq[rg * RPT + r];
      acc.x = fmaf(w, rows[r].x, acc.x);
      acc.y = fmaf(w, rows[r].y, acc.y);
      acc.z = fmaf(w, rows[r].z, acc.z);
      acc.w = fmaf(w, rows[r].w, acc.w);
      dacc = fmaf(w, zr[r], dacc);
    }
    // reduce over the row groups that share a warp (lanes CG apart)
#pragma unroll
    for (int off = CG; off < 32; off <<= 1) {
      acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
      acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
      acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
      acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
      dacc += __shfl_xor_sync(0xffffffffu, dacc, off);
    }
    static_assert(CG <= 32, "a warp must span all column groups");
    if (lane < CG) {
      *reinterpret_cast<float4*>(&s_red[warp][cg * 4]) = acc;
      if (cg == 0) s_den[warp] = dacc;
    }
    __syncthreads();
    if (tid < DV) {
      // every warp spans all DV columns (CG <= 32), so each holds a partial
      // of every column and of the denominator
      float num = 0.0f, den = a.eps;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        num += s_red[w][tid];
        den += s_den[w];
      }
      const float o = num / den;
      const size_t oi = ((size_t)b * a.Hq + (size_t)g * G + h) * DV + tid;
      if (BF16)
        static_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(o);
      else
        static_cast<float*>(a.out)[oi] = o;
    }
    __syncthreads();
  }
}

template <int D, int DV>
cudaError_t launch(const DecodeLaunch& p, cudaStream_t stream) {
  const int G = p.Hq / p.Hkv;
  const size_t smem = (size_t)G * D * sizeof(float);
  dim3 grid(p.Hkv, p.B);
  if (p.bf16) {
    auto kern = lt_decode_kernel<D, DV, true>;
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
    }
    kern<<<grid, kT, smem, stream>>>(p);
  } else {
    auto kern = lt_decode_kernel<D, DV, false>;
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
    }
    kern<<<grid, kT, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeLaunch& p, cudaStream_t stream) {
  if (p.d == 64 && p.dv == 64) return launch<64, 64>(p, stream);
  if (p.d == 128 && p.dv == 128) return launch<128, 128>(p, stream);
  if (p.d == 64 && p.dv == 128) return launch<64, 128>(p, stream);
  if (p.d == 128 && p.dv == 64) return launch<128, 64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace lt
