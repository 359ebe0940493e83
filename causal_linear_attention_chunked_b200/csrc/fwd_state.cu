// fwd_state.cu -- the forward pass continued from a given state, returning
// the final state (lineartile 1.0.0, "Features": KV-cache reuse, where the
// cache of linear attention is its fixed-size state; "Reference": the
// recurrent view of the cited linear attention).
//
// With an initial state (S0, z0) for a sequence's KV head, the outputs are
//     causal:     O_i = phi(Q_i)(S0 + S_i) / (phi(Q_i).(z0 + z_i) + eps)
//     non-causal: the same with S_i, z_i summed over the whole sequence,
// and the final state is S0 + sum over the whole sequence: splitting a
// sequence and carrying the state across the split reproduces the unsplit
// result, and the final state feeds the decode step directly.
//
// bf16 evaluation reuses the block-parallel scan ("Why Stream Wins at
// Ultra-Long Context", section 5.3, the second level over blocks).  Short
// blocks (the one-launch path of lt_linear_attn_fwd) run that single
// cooperative launch, whose carries start from S0 and whose last block also
// writes the final state; otherwise three launches:
//   1. the state launch writes the aggregate A_b of every block;
//   2. lt_state_prefix_kernel turns them, in block order, into each block's
//      carry, S0 + sum_{b' < b} A_b' (causal) or S0 + sum_b A_b (non-causal),
//      in place, and writes the final state S0 + sum_b A_b;
//   3. the forward launch starts every block from its slot.
// With S0 = 0 the carries are the very sums (same order) that the ordinary
// two-launch path forms, so the outputs are bit-identical to it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lt_internal.h"
#include "lt_fault.h"
#include "lt_state.h"

namespace lt {
namespace {

constexpr int kPrefixThreads = 256;

// One thread per element e of a lane's [S | z] (S row-major d x dv, then z),
// grid (ceil(E / 256), H_kv, sequences).  ws: [lane][nb][E].
__global__ void __launch_bounds__(kPrefixThreads)
    lt_state_prefix_kernel(float* ws, int nb, int Hkv, int d, int dv, int causal,
                           const float* s0, const float* z0, float* s_out, float* z_out) {
  const int E = d * dv + d;
  const int e = blockIdx.x * kPrefixThreads + threadIdx.x;
  if (e >= E) return;
  const size_t lane = (size_t)blockIdx.z * Hkv + blockIdx.y;
  const bool in_s = e < d * dv;
  float run = 0.0f;
  if (s0 != nullptr)
    run = in_s ? s0[lane * d * dv + e] : z0[lane * d + (e - d * dv)];
  float* w = ws + lane * (size_t)nb * E + e;
  if (causal) {
    for (int b = 0; b < nb; ++b) {  // exclusive prefix, in block order
      const float ab = w[(size_t)b * E];
      w[(size_t)b * E] = run;
      run += ab;
    }
  } else {
    for (int b = 0; b < nb; ++b) run += w[(size_t)b * E];
    for (int b = 0; b < nb; ++b) w[(size_t)b * E] = run;
  }
  if (s_out != nullptr) {
    if (in_s)
      s_out[lane * d * dv + e] = run;
    else
      z_out[lane * d + (e - d * dv)] = run;
  }
}

}  // namespace

cudaError_t launch_state_prefix(const FwdLaunch& p, int nb, float* ws, const float* s0,
                                const float* z0, float* s_out, float* z_out,
                                cudaStream_t stream) {
  const size_t E = (size_t)p.d * p.dv + p.d;
  const dim3 grid((unsigned)((E + kPrefixThreads - 1) / kPrefixThreads), p.Hkv, p.B);
  lt_state_prefix_kernel<<<grid, kPrefixThreads, 0, stream>>>(ws, nb, p.Hkv, p.d, p.dv, p.causal,
                                                              s0, z0, s_out, z_out);
  return cudaGetLastError();
}

cudaError_t launch_fwd_state(const FwdLaunch& p, bool bf16, const float* s0, const float* z0,
                             float* s_out, float* z_out, cudaStream_t stream) {
  if (!bf16) return launch_fwd_f32_state(p, s0, z0, s_out, z_out, stream);
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int nb = block_count(p, sms);  // 1 for packed sequences
  const size_t E = (size_t)p.d * p.dv + p.d;
  const size_t bytes = (size_t)p.B * p.Hkv * nb * E * sizeof(float);
  void* ws = nullptr;
  if (injected_workspace_alloc_failure()) return cudaErrorMemoryAllocation;
  cudaError_t e = cudaMallocAsync(&ws, bytes, stream);
  if (e != cudaSuccess) return e;
  if (sched_kernel() == LT_SCHED_AUTO && block_fused_supported(p, nb, sms)) {
    // short blocks: one cooperative launch that also folds in S0 and writes
    // the final state (the carries are the same sums in the same order)
    e = launch_fwd_bf16_block_fused_state(p, nb, static_cast<float*>(ws), s0, z0, s_out, z_out,
                                          stream);
    const cudaError_t f = cudaFreeAsync(ws, stream);
    return e != cudaSuccess ? e : f;
  }
  float* w = static_cast<float*>(ws);
  // 1. every block's aggregate (the state launch in its all-blocks mode)
  FwdLaunch all = p;
  all.causal = 0;
  e = launch_block_state(all, nb, w, stream);
  // 2. carries and the final state
  if (e == cudaSuccess) e = launch_state_prefix(p, nb, w, s0, z0, s_out, z_out, stream);
  // 3. the forward launch from the precomputed carries
  if (e == cudaSuccess)
    e = (p.d == 64 && p.dv == 64) ? launch_fwd_bf16_block_pre(p, nb, w, stream)
                                  : launch_fwd_bf16_seq_pre(p, nb, w, stream);
  const cudaError_t f = cudaFreeAsync(ws, stream);
  return e != cudaSuccess ? e : f;
}

}  // namespace lt
