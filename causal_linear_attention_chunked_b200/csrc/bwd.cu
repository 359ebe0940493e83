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
// backward recurrence of its section 4.2), and each cut into blocks of whole
// chunks so that every (head, block) pair runs on its own CTA:
//   0. per (sequence, KV head, block): A_b = sum_{c in b} phi(K_c)^T [V_c | 1];
//   1. forward scan per (sequence, query head, block), from the state
//      [S | z] = sum_{b' < b} A_b' (every block when non-causal): per chunk O
//      and den recomputed, g and h written to a workspace,
//          dphi(Q_c) = mask(G [V|1]^T) phi(K_c) + g S^T + h z^T,
//      and the block's sums R_b = sum phi(Q)^T g, r_b = sum phi(Q)^T h;
//   2. reverse scan per (sequence, KV head, block), from R, r = the sums of
//      the later blocks (every block when non-causal) over the group's query
//      heads:
//          dphi(K_c) = V_c R^T + r + sum_h mask(G [V|1]^T)^T phi(Q_c),
//          dV_c      = phi(K_c) R  + sum_h mask(phi(Q) phi(K)^T)^T g,
//      R, r gaining each chunk's phi(Q)^T [g | h] (causal).
// Non-causal: no chunk-local terms.  The block sums are added in block
// order (query heads in order), so the results do not depend on scheduling.
// fp32 FMA arithmetic on shared-memory tiles, each thread holding a small
// register tile of every product (bf16 or fp32 inputs and outputs, outputs
// rounded once).  Workspace: g and h for every (token, query head) and the
// two sets of block sums.
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
constexpr int kT = 256;  // threads per CTA: 16 row groups x 16 column groups

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
  float* gws;  // g = dout / den      [tokens][Hq][dv]
  float* hws;  // h                   [tokens][Hq]
  float* akv;  // block sums phi(K)^T [V | 1]  [B][Hkv][nb][d*dv + d]
  float* aqg;  // block sums phi(Q)^T [g | h]  [B][Hq][nb][d*dv + d]
  const int32_t* cu_seqlens;
  int Hq, Hkv, N, causal;
  int nb;  // blocks per sequence (the grid's y extent)
  int lb;  // tokens per block, a multiple of kC
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

// Shared tiles are row-major with one float of padding per row: a warp
// walking a column (rows varying) or a row (columns varying) touches 32
// different banks.
// rows [c0, c0 + kC) of head h of a token-major [.][H][W] tensor -> dst
// [kC][W + 1] fp32 (phi applied when `phi`); rows past n are zero
template <typename T, int W>
__device__ __forceinline__ void load_tile(float (*dst)[W + 1], const T* src, int t0, int c0, int n,
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

// ---------------------------------------------------------------- pass A
// phi(K)^T [V | 1] of each block: thread (ig, cg) of the 16 x 16 grid holds
// rows ig + 16m, columns cg + 16n of the [d][dv] sum (and z for cg == 0).
template <typename T, int D, int DV>
struct SmA {
  float pk[kC][D + 1];
  float vv[kC][DV + 1];
};

template <typename T, int D, int DV>
__global__ void __launch_bounds__(kT) lt_bwd_kvsum_kernel(const BwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SmA<T, D, DV>& sm = *reinterpret_cast<SmA<T, D, DV>*>(smem_raw);
  constexpr int MR = D / 16, NC = DV / 16, E = D * DV + D;
  const int tid = threadIdx.x, g = blockIdx.x, b = blockIdx.y, s = blockIdx.z;
  const int ig = tid >> 4, cg = tid & 15;
  int t0, n;
  if (!seq_of(a, s, t0, n)) {
    if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
    return;
  }
  const int lo = b * a.lb;
  if (lo >= n) return;
  const int hi = min(n, lo + a.lb);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  float S[MR][NC], z[MR];
#pragma unroll
  for (int m = 0; m < MR; ++m) {
    z[m] = 0.0f;
#pragma unroll
    for (int c = 0; c < NC; ++c) S[m][c] = 0.0f;
  }
  for (int c0 = lo; c0 < hi; c0 += kC) {
    load_tile<T, D>(sm.pk, k, t0, c0, n, a.Hkv, g, true);
    load_tile<T, DV>(sm.vv, v, t0, c0, n, a.Hkv, g, false);
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < kC; ++j) {
      float vj[NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) vj[c] = sm.vv[j][cg + 16 * c];
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        const float p = sm.pk[j][ig + 16 * m];
        z[m] += p;
#pragma unroll
        for (int c = 0; c < NC; ++c) S[m][c] = fmaf(p, vj[c], S[m][c]);
      }
    }
    __syncthreads();
  }
  float* dst = a.akv + (((size_t)s * a.Hkv + g) * a.nb + b) * E;
#pragma unroll
  for (int m = 0; m < MR; ++m) {
#pragma unroll
    for (int c = 0; c < NC; ++c) dst[(ig + 16 * m) * DV + cg + 16 * c] = S[m][c];
    if (cg == 0) dst[D * DV + ig + 16 * m] = z[m];
  }
}

// sum of the [E] block sums src[i * stride] for i in [i0, i1) (in that
// order) -> dst (the [d][dv + 1]-padded state and its d-vector)
template <int D, int DV>
__device__ __forceinline__ void sum_blocks(float (*S)[DV + 1], float* z, const float* src,
                                           size_t stride, int i0, int i1) {
  constexpr int E = D * DV + D, PER = (E + kT - 1) / kT;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
  for (int i = i0; i < i1; ++i) {
    const float* p = src + (size_t)i * stride;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int x = threadIdx.x + e * kT;
      if (x < E) acc[e] += __ldcg(p + x);
    }
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int x = threadIdx.x + e * kT;
    if (x < D * DV)
      S[x / DV][x % DV] = acc[e];
    else if (x < E)
      z[x - D * DV] = acc[e];
  }
}

// ---------------------------------------------------------------- kernel 1
template <typename T, int D, int DV>
struct Sm1 {
  float S[D][DV + 1];
  float z[D];
  float pq[kC][D + 1];
  float pk[kC][D + 1];
  float vv[kC][DV + 1];
  float gg[kC][DV + 1];  // dO, then g
  float A[kC][kC + 1];   // masked scores, then masked da
  float den[kC];
  float hh[kC];
};

// One CTA per (query head, block, sequence).  Thread (ig, cg): rows 2ig and
// 2ig + 1 of the chunk's [32][.] products, columns cg + 16n; rows ig + 16m,
// columns cg + 16n of the [d][dv] ones.
template <typename T, int D, int DV>
__global__ void __launch_bounds__(kT) lt_bwd_dq_kernel(const BwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Sm1<T, D, DV>& sm = *reinterpret_cast<Sm1<T, D, DV>*>(smem_raw);
  constexpr int MR = D / 16, NC = DV / 16, ND = D / 16, E = D * DV + D;
  const int tid = threadIdx.x, h = blockIdx.x, b = blockIdx.y, s = blockIdx.z;
  const int ig = tid >> 4, cg = tid & 15, warp = tid >> 5, lane = tid & 31;
  const int i0 = 2 * ig, i1 = i0 + 1;
  const int G = a.Hq / a.Hkv, g = h / G;
  int t0, n;
  if (!seq_of(a, s, t0, n)) {
    if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
    return;
  }
  const int lo = b * a.lb;
  if (lo >= n) return;
  const int hi = min(n, lo + a.lb), nblk = (n + a.lb - 1) / a.lb;
  const bool causal = a.causal != 0;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  const T* dout = static_cast<const T*>(a.dout);
  T* dq = static_cast<T*>(a.dq);
  // the state of the earlier blocks (causal) or of the whole sequence
  sum_blocks<D, DV>(sm.S, sm.z, a.akv + ((size_t)s * a.Hkv + g) * a.nb * E, E, 0,
                    causal ? b : nblk);
  float R[MR][NC], r[MR];  // this block's phi(Q)^T [g | h]
#pragma unroll
  for (int m = 0; m < MR; ++m) {
    r[m] = 0.0f;
#pragma unroll
    for (int c = 0; c < NC; ++c) R[m][c] = 0.0f;
  }
  __syncthreads();
  for (int c0 = lo; c0 < hi; c0 += kC) {
    load_tile<T, D>(sm.pq, q, t0, c0, n, a.Hq, h, true);
    load_tile<T, D>(sm.pk, k, t0, c0, n, a.Hkv, g, true);
    load_tile<T, DV>(sm.vv, v, t0, c0, n, a.Hkv, g, false);
    load_tile<T, DV>(sm.gg, dout, t0, c0, n, a.Hq, h, false);
    __syncthreads();
    if (causal) {  // masked chunk scores: rows i0, i1; columns cg, cg + 16
      float x[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 8
      for (int e = 0; e < D; ++e) {
        const float p0 = sm.pq[i0][e], p1 = sm.pq[i1][e];
        const float k0 = sm.pk[cg][e], k1 = sm.pk[cg + 16][e];
        x[0][0] = fmaf(p0, k0, x[0][0]);
        x[0][1] = fmaf(p0, k1, x[0][1]);
        x[1][0] = fmaf(p1, k0, x[1][0]);
        x[1][1] = fmaf(p1, k1, x[1][1]);
      }
      sm.A[i0][cg] = cg <= i0 ? x[0][0] : 0.0f;
      sm.A[i0][cg + 16] = cg + 16 <= i0 ? x[0][1] : 0.0f;
      sm.A[i1][cg] = cg <= i1 ? x[1][0] : 0.0f;
      sm.A[i1][cg + 16] = cg + 16 <= i1 ? x[1][1] : 0.0f;
      __syncthreads();
    }
    // den: warp w takes rows 4w .. 4w + 3
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int i = 4 * warp + rr;
      float x = causal ? sm.A[i][lane] : 0.0f;
#pragma unroll
      for (int e = lane; e < D; e += 32) x = fmaf(sm.pq[i][e], sm.z[e], x);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (lane == 0) sm.den[i] = x + a.eps;
    }
    __syncthreads();
    // numerator rows i0, i1 (columns cg + 16c), then O, g and h
    {
      float o[2][NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) o[0][c] = o[1][c] = 0.0f;
      if (causal) {
#pragma unroll 4
        for (int j = 0; j < kC; ++j) {
          const float a0 = sm.A[i0][j], a1 = sm.A[i1][j];
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            const float vj = sm.vv[j][cg + 16 * c];
            o[0][c] = fmaf(a0, vj, o[0][c]);
            o[1][c] = fmaf(a1, vj, o[1][c]);
          }
        }
      }
#pragma unroll 4
      for (int e = 0; e < D; ++e) {
        const float p0 = sm.pq[i0][e], p1 = sm.pq[i1][e];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const float sv = sm.S[e][cg + 16 * c];
          o[0][c] = fmaf(p0, sv, o[0][c]);
          o[1][c] = fmaf(p1, sv, o[1][c]);
        }
      }
      // rows past the end get g = h = 0 (their den is eps, possibly 0)
      const float inv0 = c0 + i0 < n ? 1.0f / sm.den[i0] : 0.0f;
      const float inv1 = c0 + i1 < n ? 1.0f / sm.den[i1] : 0.0f;
      float dot0 = 0.0f, dot1 = 0.0f;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const float d0 = sm.gg[i0][cg + 16 * c], d1 = sm.gg[i1][cg + 16 * c];
        dot0 = fmaf(d0, o[0][c] * inv0, dot0);
        dot1 = fmaf(d1, o[1][c] * inv1, dot1);
        sm.gg[i0][cg + 16 * c] = d0 * inv0;
        sm.gg[i1][cg + 16 * c] = d1 * inv1;
      }
#pragma unroll
      for (int o2 = 8; o2 > 0; o2 >>= 1) {  // the 16 threads of row group ig
        dot0 += __shfl_xor_sync(0xffffffffu, dot0, o2);
        dot1 += __shfl_xor_sync(0xffffffffu, dot1, o2);
      }
      if (cg == 0) {
        sm.hh[i0] = -dot0 * inv0;
        sm.hh[i1] = -dot1 * inv1;
      }
      // g and h to the workspace (the dk, dv launch reads them)
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int i = i0 + m;
        if (c0 + i < n) {
          const size_t row = (size_t)(t0 + c0 + i) * a.Hq + h;
#pragma unroll
          for (int c = 0; c < NC; ++c) a.gws[row * DV + cg + 16 * c] = sm.gg[i][cg + 16 * c];
          if (cg == 0) a.hws[row] = -(m ? dot1 * inv1 : dot0 * inv0);
        }
      }
    }
    __syncthreads();
    if (causal) {  // masked da (overwrites the scores)
      float x[2][2];
      x[0][0] = x[0][1] = sm.hh[i0];
      x[1][0] = x[1][1] = sm.hh[i1];
#pragma unroll 8
      for (int c = 0; c < DV; ++c) {
        const float g0 = sm.gg[i0][c], g1 = sm.gg[i1][c];
        const float v0 = sm.vv[cg][c], v1 = sm.vv[cg + 16][c];
        x[0][0] = fmaf(g0, v0, x[0][0]);
        x[0][1] = fmaf(g0, v1, x[0][1]);
        x[1][0] = fmaf(g1, v0, x[1][0]);
        x[1][1] = fmaf(g1, v1, x[1][1]);
      }
      sm.A[i0][cg] = cg <= i0 ? x[0][0] : 0.0f;
      sm.A[i0][cg + 16] = cg + 16 <= i0 ? x[0][1] : 0.0f;
      sm.A[i1][cg] = cg <= i1 ? x[1][0] : 0.0f;
      sm.A[i1][cg + 16] = cg + 16 <= i1 ? x[1][1] : 0.0f;
      __syncthreads();
    }
    // dphi(Q) = da phi(K) + g S^T + h z^T;  dQ = dphi(Q) * min(phi(Q), 1)
    {
      float x[2][ND];
#pragma unroll
      for (int c = 0; c < ND; ++c) {
        const float zc = sm.z[cg + 16 * c];
        x[0][c] = sm.hh[i0] * zc;
        x[1][c] = sm.hh[i1] * zc;
      }
      if (causal) {
#pragma unroll 4
        for (int j = 0; j < kC; ++j) {
          const float d0 = sm.A[i0][j], d1 = sm.A[i1][j];
#pragma unroll
          for (int c = 0; c < ND; ++c) {
            const float kj = sm.pk[j][cg + 16 * c];
            x[0][c] = fmaf(d0, kj, x[0][c]);
            x[1][c] = fmaf(d1, kj, x[1][c]);
          }
        }
      }
#pragma unroll 4
      for (int e = 0; e < DV; ++e) {
        const float g0 = sm.gg[i0][e], g1 = sm.gg[i1][e];
#pragma unroll
        for (int c = 0; c < ND; ++c) {
          const float sv = sm.S[cg + 16 * c][e];
          x[0][c] = fmaf(g0, sv, x[0][c]);
          x[1][c] = fmaf(g1, sv, x[1][c]);
        }
      }
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int i = i0 + m;
        if (c0 + i < n) {
          T* row = dq + ((size_t)(t0 + c0 + i) * a.Hq + h) * D;
#pragma unroll
          for (int c = 0; c < ND; ++c)
            from_f(row + cg + 16 * c, x[m][c] * fminf(sm.pq[i][cg + 16 * c], 1.0f));
        }
      }
    }
    // this block's phi(Q)^T [g | h]
#pragma unroll 4
    for (int i = 0; i < kC; ++i) {
      float gi[NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) gi[c] = sm.gg[i][cg + 16 * c];
      const float hi_ = sm.hh[i];
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        const float p = sm.pq[i][ig + 16 * m];
        r[m] = fmaf(p, hi_, r[m]);
#pragma unroll
        for (int c = 0; c < NC; ++c) R[m][c] = fmaf(p, gi[c], R[m][c]);
      }
    }
    if (causal && c0 + kC < hi) {  // the state after this chunk
      __syncthreads();  // every read of S is done
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        const int e = ig + 16 * m;
        float x[NC], zs = 0.0f;
#pragma unroll
        for (int c = 0; c < NC; ++c) x[c] = sm.S[e][cg + 16 * c];
#pragma unroll 4
        for (int j = 0; j < kC; ++j) {
          const float p = sm.pk[j][e];
          zs += p;
#pragma unroll
          for (int c = 0; c < NC; ++c) x[c] = fmaf(p, sm.vv[j][cg + 16 * c], x[c]);
        }
#pragma unroll
        for (int c = 0; c < NC; ++c) sm.S[e][cg + 16 * c] = x[c];
        if (cg == 0) sm.z[e] += zs;
      }
    }
    __syncthreads();
  }
  float* dst = a.aqg + (((size_t)s * a.Hq + h) * a.nb + b) * E;
#pragma unroll
  for (int m = 0; m < MR; ++m) {
#pragma unroll
    for (int c = 0; c < NC; ++c) dst[(ig + 16 * m) * DV + cg + 16 * c] = R[m][c];
    if (cg == 0) dst[D * DV + ig + 16 * m] = r[m];
  }
}

// ---------------------------------------------------------------- kernel 2
template <typename T, int D, int DV>
struct Sm2 {
  float R[D][DV + 1];
  float r[D];
  float pk[kC][D + 1];
  float vv[kC][DV + 1];
  float pq[kC][D + 1];
  float gg[kC][DV + 1];
  float hh[kC];
  float A[kC][kC + 1];
  float dA[kC][kC + 1];
};

// One CTA per (KV head, block, sequence), chunks in reverse order.  Thread
// (ig, cg): rows 2ig, 2ig + 1 of the chunk's dk, dv; rows ig + 16m,
// columns cg + 16n of R.
template <typename T, int D, int DV>
__global__ void __launch_bounds__(kT) lt_bwd_dkv_kernel(const BwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Sm2<T, D, DV>& sm = *reinterpret_cast<Sm2<T, D, DV>*>(smem_raw);
  constexpr int MR = D / 16, NC = DV / 16, ND = D / 16, E = D * DV + D;
  const int tid = threadIdx.x, g = blockIdx.x, b = blockIdx.y, s = blockIdx.z;
  const int ig = tid >> 4, cg = tid & 15;
  const int j0 = 2 * ig, j1 = j0 + 1;
  const int G = a.Hq / a.Hkv;
  int t0, n;
  if (!seq_of(a, s, t0, n)) {
    if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
    return;
  }
  const int lo = b * a.lb;
  if (lo >= n) return;
  const int hi = min(n, lo + a.lb), nblk = (n + a.lb - 1) / a.lb;
  const bool causal = a.causal != 0;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  T* dk = static_cast<T*>(a.dk);
  T* dvo = static_cast<T*>(a.dv);
  // R, r of the later blocks (causal) or of the whole sequence, over the
  // group's query heads in order
  {
    constexpr int PER = (E + kT - 1) / kT;
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
    for (int hq = g * G; hq < (g + 1) * G; ++hq) {
      const float* src = a.aqg + ((size_t)s * a.Hq + hq) * a.nb * E;
      for (int i = causal ? b + 1 : 0; i < nblk; ++i) {
        const float* p = src + (size_t)i * E;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          const int x = tid + e * kT;
          if (x < E) acc[e] += __ldcg(p + x);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int x = tid + e * kT;
      if (x < D * DV)
        sm.R[x / DV][x % DV] = acc[e];
      else if (x < E)
        sm.r[x - D * DV] = acc[e];
    }
  }
  __syncthreads();
  float Rr[MR][NC], rr[MR];  // this thread's part of R, r (causal: updated per chunk)
#pragma unroll
  for (int m = 0; m < MR; ++m) {
    rr[m] = sm.r[ig + 16 * m];
#pragma unroll
    for (int c = 0; c < NC; ++c) Rr[m][c] = sm.R[ig + 16 * m][cg + 16 * c];
  }
  const int nch = (hi - lo + kC - 1) / kC;
  for (int ci = nch - 1; ci >= 0; --ci) {
    const int c0 = lo + ci * kC;
    load_tile<T, D>(sm.pk, k, t0, c0, n, a.Hkv, g, true);
    load_tile<T, DV>(sm.vv, v, t0, c0, n, a.Hkv, g, false);
    __syncthreads();
    // the later chunks (causal) or the whole sequence, through R, r:
    //   dphi(K)_j = V_j R^T + r,  dV_j = phi(K)_j R
    float xk[2][ND], xv[2][NC];
#pragma unroll
    for (int c = 0; c < ND; ++c) xk[0][c] = xk[1][c] = sm.r[cg + 16 * c];
#pragma unroll
    for (int c = 0; c < NC; ++c) xv[0][c] = xv[1][c] = 0.0f;
#pragma unroll 4
    for (int e = 0; e < DV; ++e) {
      const float v0 = sm.vv[j0][e], v1 = sm.vv[j1][e];
#pragma unroll
      for (int c = 0; c < ND; ++c) {
        const float rv = sm.R[cg + 16 * c][e];
        xk[0][c] = fmaf(v0, rv, xk[0][c]);
        xk[1][c] = fmaf(v1, rv, xk[1][c]);
      }
    }
#pragma unroll 4
    for (int e = 0; e < D; ++e) {
      const float k0 = sm.pk[j0][e], k1 = sm.pk[j1][e];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const float rv = sm.R[e][cg + 16 * c];
        xv[0][c] = fmaf(k0, rv, xv[0][c]);
        xv[1][c] = fmaf(k1, rv, xv[1][c]);
      }
    }
    if (causal) {
      // the chunk itself, every query head of the group; R, r gain the chunk
      for (int hq = g * G; hq < (g + 1) * G; ++hq) {
        load_tile<T, D>(sm.pq, q, t0, c0, n, a.Hq, hq, true);
        for (int e = tid; e < kC * DV; e += kT) {
          const int i = e / DV, c = e % DV;
          sm.gg[i][c] = c0 + i < n ? a.gws[((size_t)(t0 + c0 + i) * a.Hq + hq) * DV + c] : 0.0f;
        }
        if (tid < kC) sm.hh[tid] = c0 + tid < n ? a.hws[(size_t)(t0 + c0 + tid) * a.Hq + hq] : 0.0f;
        __syncthreads();
        {  // rows i = 2ig, 2ig + 1; columns j = cg, cg + 16
          const int r0 = j0, r1 = j1;
          float x[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
          float y[2][2];
          y[0][0] = y[0][1] = sm.hh[r0];
          y[1][0] = y[1][1] = sm.hh[r1];
#pragma unroll 8
          for (int e = 0; e < D; ++e) {
            const float p0 = sm.pq[r0][e], p1 = sm.pq[r1][e];
            const float k0 = sm.pk[cg][e], k1 = sm.pk[cg + 16][e];
            x[0][0] = fmaf(p0, k0, x[0][0]);
            x[0][1] = fmaf(p0, k1, x[0][1]);
            x[1][0] = fmaf(p1, k0, x[1][0]);
            x[1][1] = fmaf(p1, k1, x[1][1]);
          }
#pragma unroll 8
          for (int e = 0; e < DV; ++e) {
            const float g0 = sm.gg[r0][e], g1 = sm.gg[r1][e];
            const float v0 = sm.vv[cg][e], v1 = sm.vv[cg + 16][e];
            y[0][0] = fmaf(g0, v0, y[0][0]);
            y[0][1] = fmaf(g0, v1, y[0][1]);
            y[1][0] = fmaf(g1, v0, y[1][0]);
            y[1][1] = fmaf(g1, v1, y[1][1]);
          }
          sm.A[r0][cg] = cg <= r0 ? x[0][0] : 0.0f;
          sm.A[r0][cg + 16] = cg + 16 <= r0 ? x[0][1] : 0.0f;
          sm.A[r1][cg] = cg <= r1 ? x[1][0] : 0.0f;
          sm.A[r1][cg + 16] = cg + 16 <= r1 ? x[1][1] : 0.0f;
          sm.dA[r0][cg] = cg <= r0 ? y[0][0] : 0.0f;
          sm.dA[r0][cg + 16] = cg + 16 <= r0 ? y[0][1] : 0.0f;
          sm.dA[r1][cg] = cg <= r1 ? y[1][0] : 0.0f;
          sm.dA[r1][cg + 16] = cg + 16 <= r1 ? y[1][1] : 0.0f;
        }
        __syncthreads();
        // dphi(K)_j += sum_i da_ij phi(Q)_i,  dV_j += sum_i a_ij g_i (i >= j)
#pragma unroll 4
        for (int i = 0; i < kC; ++i) {
          const float d0 = sm.dA[i][j0], d1 = sm.dA[i][j1];
          const float a0 = sm.A[i][j0], a1 = sm.A[i][j1];
#pragma unroll
          for (int c = 0; c < ND; ++c) {
            const float p = sm.pq[i][cg + 16 * c];
            xk[0][c] = fmaf(d0, p, xk[0][c]);
            xk[1][c] = fmaf(d1, p, xk[1][c]);
          }
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            const float gv = sm.gg[i][cg + 16 * c];
            xv[0][c] = fmaf(a0, gv, xv[0][c]);
            xv[1][c] = fmaf(a1, gv, xv[1][c]);
          }
        }
        // R += phi(Q)^T g, r += phi(Q)^T h
#pragma unroll 4
        for (int i = 0; i < kC; ++i) {
          float gi[NC];
#pragma unroll
          for (int c = 0; c < NC; ++c) gi[c] = sm.gg[i][cg + 16 * c];
          const float hv = sm.hh[i];
#pragma unroll
          for (int m = 0; m < MR; ++m) {
            const float p = sm.pq[i][ig + 16 * m];
            rr[m] = fmaf(p, hv, rr[m]);
#pragma unroll
            for (int c = 0; c < NC; ++c) Rr[m][c] = fmaf(p, gi[c], Rr[m][c]);
          }
        }
        __syncthreads();
      }
      // R, r for the earlier chunks (every read of the old values is done:
      // the group loop above passed a barrier after them)
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        if (cg == 0) sm.r[ig + 16 * m] = rr[m];
#pragma unroll
        for (int c = 0; c < NC; ++c) sm.R[ig + 16 * m][cg + 16 * c] = Rr[m][c];
      }
    }
    // dK = dphi(K) * min(phi(K), 1); dV
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int j = j0 + m;
      if (c0 + j < n) {
        T* rk = dk + ((size_t)(t0 + c0 + j) * a.Hkv + g) * D;
        T* rv = dvo + ((size_t)(t0 + c0 + j) * a.Hkv + g) * DV;
#pragma unroll
        for (int c = 0; c < ND; ++c)
          from_f(rk + cg + 16 * c, xk[m][c] * fminf(sm.pk[j][cg + 16 * c], 1.0f));
#pragma unroll
        for (int c = 0; c < NC; ++c) from_f(rv + cg + 16 * c, xv[m][c]);
      }
    }
    __syncthreads();
  }
}

template <typename T, int D, int DV>
cudaError_t launch_bwd_t(const BwdArgs& a, int B, cudaStream_t stream) {
  const size_t s0 = sizeof(SmA<T, D, DV>), s1 = sizeof(Sm1<T, D, DV>),
               s2 = sizeof(Sm2<T, D, DV>);
  auto k0 = lt_bwd_kvsum_kernel<T, D, DV>;
  auto k1 = lt_bwd_dq_kernel<T, D, DV>;
  auto k2 = lt_bwd_dkv_kernel<T, D, DV>;
  cudaError_t e = cudaFuncSetAttribute(k0, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s0);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
  if (e != cudaSuccess) return e;
  k0<<<dim3(a.Hkv, a.nb, B), kT, s0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k1<<<dim3(a.Hq, a.nb, B), kT, s1, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k2<<<dim3(a.Hkv, a.nb, B), kT, s2, stream>>>(a);
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
  // blocks per sequence: about four CTAs per SM in the KV-head launches (two
  // and eight measured slower at B2 H8 N4096 d64, at B2 Hq32 Hkv8 N16384 d128
  // and at B1 H8 N65536 d64)
  const int sms = lt::device_sm_count();
  if (sms <= 0) return LT_ERR_CUDA;
  const long long lanes = (long long)B * H_kv;
  const long long nch = (N + 31) / 32;  // chunks of the longest possible sequence
  long long nb = (4LL * sms + lanes - 1) / lanes;
  if (nb > nch) nb = nch;
  if (nb < 1) nb = 1;
  const long long lb = ((N + nb - 1) / nb + 31) / 32 * 32;
  nb = (N + lb - 1) / lb;
  const size_t E = (size_t)d * dv_w + d;
  const size_t n_g = (size_t)T * H_q * dv_w, n_h = (size_t)T * H_q;
  const size_t n_kv = (size_t)B * H_kv * nb * E, n_qg = (size_t)B * H_q * nb * E;
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, (n_g + n_h + n_kv + n_qg) * sizeof(float), (cudaStream_t)stream) !=
      cudaSuccess) {
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
  a.gws = static_cast<float*>(ws);
  a.hws = a.gws + n_g;
  a.akv = a.hws + n_h;
  a.aqg = a.akv + n_kv;
  a.cu_seqlens = cu_seqlens;
  a.Hq = H_q;
  a.Hkv = H_kv;
  a.N = N;
  a.causal = causal;
  a.nb = (int)nb;
  a.lb = (int)lb;
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
