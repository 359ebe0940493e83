// lt_state.h -- internal launchers of the forward pass continued from a given
// state and returning the final state (prefill -> decode handoff, chunked
// continuation).  The state of a (sequence, KV head) is S [d][dv] and z [d]
// in fp32, laid out [sequence][KV head][.] as the decode step takes it.
#pragma once
#include <cuda_runtime.h>

#include "lt_internal.h"

namespace lt {

// The bf16 forward launches with a precomputed carry: slot b of the lane's
// workspace already holds block b's carry (no summing of earlier
// aggregates), and every block, the first included, starts from it.
cudaError_t launch_fwd_bf16_block_pre(const FwdLaunch& p, int nb, const float* ws,
                                      cudaStream_t stream);
cudaError_t launch_fwd_bf16_seq_pre(const FwdLaunch& p, int nb, const float* ws,
                                    cudaStream_t stream);

// fp32 forward from the state (s0, z0) (nullptr: zero), writing the final
// state to (s_out, z_out) (nullptr: not returned).
cudaError_t launch_fwd_f32_state(const FwdLaunch& p, const float* s0, const float* z0,
                                 float* s_out, float* z_out, cudaStream_t stream);

// The stateful forward pass for either dtype.  bf16 allocates a stream-ordered
// workspace of (sequences x H_kv x blocks) block states, (d*dv + d) floats each.
cudaError_t launch_fwd_state(const FwdLaunch& p, bool bf16, const float* s0, const float* z0,
                             float* s_out, float* z_out, cudaStream_t stream);

// Block states [lane][nb][d*dv + d] (the state launch's workspace) -> each
// block's carry in place (causal: S0 + earlier blocks; non-causal: S0 + all)
// and the final state S0 + all blocks into (s_out, z_out) (nullptr: not
// written).  p.causal selects the carry.
cudaError_t launch_state_prefix(const FwdLaunch& p, int nb, float* ws, const float* s0,
                                const float* z0, float* s_out, float* z_out,
                                cudaStream_t stream);

// The final state alone, S0 + sum over each sequence (no outputs; q unused).
cudaError_t launch_state_only(const FwdLaunch& p, bool bf16, const float* s0, const float* z0,
                              float* s_out, float* z_out, cudaStream_t stream);

}  // namespace lt
