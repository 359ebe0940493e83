// lt_internal.h -- launch descriptors shared by the C ABI layer and the
// kernel translation units (host side only).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lt_linear_attn.h"

namespace lt {

struct FwdLaunch {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  const int32_t* cu_seqlens;  // device, B+1 entries, or nullptr (dense)
  int B, Hq, Hkv, N, d, dv, causal;
  float eps;
  long long total_tokens;  // B*N (dense) or N (packed)
  int* err;                // device error word
  int in_f16;              // 1: fp16 inputs and output (bf16 tensor-core operands)
  int phi;                 // feature map (lt_feature_map_t); 0 = ELU + 1
};

struct DecodeLaunch {
  const void* q;
  const void* k;
  const void* v;
  float* S;
  float* z;
  void* out;
  int B, Hq, Hkv, d, dv;
  float eps;
  int bf16;  // 1: bf16 q/k/v/out, 0: fp32
};

// bf16 forward: picks the block count, allocates the block workspace
// (stream-ordered) and runs the state launch then the forward launch
cudaError_t launch_fwd_bf16(const FwdLaunch& p, cudaStream_t stream);
// what launch_fwd_bf16 does for p on a device with num_sms SMs: blocks per
// sequence, kernel launches, workspace bytes
void plan_fwd_bf16(const FwdLaunch& p, int num_sms, int* nb, int* launches, size_t* ws_bytes);
// the same with a caller-provided workspace of at least
// block_workspace_bytes(p, nb) bytes (nullptr when that is 0)
cudaError_t launch_fwd_bf16_ws(const FwdLaunch& p, int nb, float* ws, cudaStream_t stream);
// Block-parallel scan.  A dense sequence is cut into nb blocks of
// block_chunks(p, nb) chunks; the state launch writes each block's aggregate
// phi(K)^T [V | 1] (fp32, d x dv then d) to the workspace and the forward
// launch starts block b from the sum of the aggregates before it (causal) or
// of all of them (non-causal).  nb = 1: no workspace, no state launch.
int block_count(const FwdLaunch& p, int num_sms);
int block_chunks(const FwdLaunch& p, int nb);
size_t block_workspace_bytes(const FwdLaunch& p, int nb);
cudaError_t launch_block_state(const FwdLaunch& p, int nb, float* ws, cudaStream_t stream);
// forward launches: d = dv = 64 specialised kernel (the carry, when nb > 1,
// from the state launch's aggregates); every width pair
bool block_supported(const FwdLaunch& p);
cudaError_t launch_fwd_bf16_block(const FwdLaunch& p, int nb, const float* ws,
                                  cudaStream_t stream);
cudaError_t launch_fwd_bf16_seq(const FwdLaunch& p, int nb, const float* ws,
                                cudaStream_t stream);
// d = dv = 64, dense, blocks of at most 4 chunks, one CTA per SM: one
// cooperative launch in which every block publishes its aggregate to the
// workspace, the CTAs meet at a grid barrier, and each block gathers its
// carry from the others (the workspace of the two-launch path)
bool block_fused_supported(const FwdLaunch& p, int nb, int num_sms);
cudaError_t launch_fwd_bf16_block_fused(const FwdLaunch& p, int nb, float* ws,
                                        cudaStream_t stream);
// the same continued from the state (s0, z0) (nullptr: zero) and writing the
// final state to (s_out, z_out) (nullptr: not returned)
cudaError_t launch_fwd_bf16_block_fused_state(const FwdLaunch& p, int nb, float* ws,
                                              const float* s0, const float* z0, float* s_out,
                                              float* z_out, cudaStream_t stream);
// the per-device error word of the current device (looked up once per device)
int* device_error_word_current();
// SM count of the current device (queried once per device); 0 on failure
int device_sm_count();
// the schedule override of lt_debug_set_schedule (LT_SCHED_AUTO and 0 unless
// a test or an ablation set them)
int sched_kernel();
int sched_blocks();
// the argument checks every forward entry point makes, in order; on LT_OK
// *p describes the call (its err field still unset)
lt_status_t check_fwd(const void* q, const void* k, const void* v, void* out, int B, int H_q,
                      int H_kv, int N, int d, int dv, int causal, float eps,
                      const int32_t* cu_seqlens, lt_dtype_t dtype, FwdLaunch* p);
cudaError_t launch_fwd_f32(const FwdLaunch& p, cudaStream_t stream);
cudaError_t launch_decode(const DecodeLaunch& p, cudaStream_t stream);

}  // namespace lt
