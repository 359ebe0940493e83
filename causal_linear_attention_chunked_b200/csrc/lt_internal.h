// lt_internal.h -- launch descriptors shared by the C ABI layer and the
// kernel translation units (host side only).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

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

cudaError_t launch_fwd_bf16(const FwdLaunch& p, cudaStream_t stream);
// d = dv = 64: sequence split over a thread-block cluster (or one CTA per
// (sequence, KV head) for packed inputs)
bool split_supported(const FwdLaunch& p);
cudaError_t launch_fwd_bf16_split(const FwdLaunch& p, cudaStream_t stream);
// d = dv = 64: block-parallel two-launch scan (block aggregates, then one CTA
// per block); `ws` holds block_workspace_bytes(p, nb) bytes when nb > 1
bool block_supported(const FwdLaunch& p);
int block_count(const FwdLaunch& p, int num_sms);
size_t block_workspace_bytes(const FwdLaunch& p, int nb);
cudaError_t launch_fwd_bf16_block(const FwdLaunch& p, int nb, float* ws, cudaStream_t stream);
cudaError_t launch_fwd_f32(const FwdLaunch& p, cudaStream_t stream);
cudaError_t launch_decode(const DecodeLaunch& p, cudaStream_t stream);

}  // namespace lt
