// state_bf16_sm100.cu -- block aggregates of the chunked linear-attention
// state, the first launch of the block-parallel forward pass (bf16 inputs,
// fp32 accumulation, sm_100a tensor cores).
//
// A sequence of n tokens is cut into nb blocks of bc chunks of 128 tokens.
// For block b this kernel computes
//     A_b = sum_{c in b} phi(K_c)^T [V_c | 1]     (d x (dv + 1), fp32)
// i.e. the block's contribution to the state S and normaliser z of the
// linear attention of lineartile 1.0.0 ("How It Works"/"Reference"), the
// chunk-local reduction of the two-level scan in "Why Stream Wins at
// Ultra-Long Context", section 5.3.  The forward launch then starts block b
// from sum_{b' < b} A_b' (causal) or sum_b A_b (non-causal).
//
// One CTA per (block, KV head, sequence); 320 threads: warps 0-7 apply phi
// to the TMA-loaded K tiles (tail rows zeroed; two warps per SM
// sub-partition) and warps 0-3 store the result, warp 8 is the TMA producer,
// warp 9 allocates TMEM and issues the MMAs that accumulate A_b in TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include "fwd_common.cuh"
#include "lt_internal.h"
#include "lt_ptx.cuh"

namespace lt {
namespace {
using namespace fwd;

constexpr int kThreads = 320;
constexpr int kXf = 256;  // transform threads

template <int D, int DV>
struct SCfg {
  static constexpr int KT = kChunk * D * 2, VT = kChunk * DV * 2, KVT = KT + VT;
  static constexpr int ONEST = kChunk * kRowBytes;
  static constexpr int NS = (KVT <= 48 * 1024) ? 4 : 3;  // K/V stages
  static constexpr int OFF_ONES = NS * KVT;
  static constexpr int OFF_BAR = OFF_ONES + ONEST;
  static constexpr int SMEM = OFF_BAR + (3 * NS + 2) * 8 + 16 + 1024;
  static constexpr int E = D * DV + D;
  static constexpr int TM_COLS = (DV + 16 <= 128) ? 128 : 256;
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct StateArgs {
  const int32_t* cu_seqlens;
  float* ws;
  int Hkv, N, nb, bc, total_tokens;
  int* err;
};

template <int D, int DV, class VAR>
__global__ void __launch_bounds__(kThreads, 1)
    lt_block_state_kernel(const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const StateArgs a) {
  using K = SCfg<D, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ volatile int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int blk = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  int t0, ntok;
  if (a.cu_seqlens) {
    const int lo = a.cu_seqlens[s], hi = a.cu_seqlens[s + 1];
    if (lo < 0 || hi < lo || hi > a.total_tokens) {
      if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
      return;
    }
    t0 = lo;
    ntok = hi - lo;
  } else {
    t0 = s * a.N;
    ntok = a.N;
  }
  const int nc = (ntok + kChunk - 1) / kChunk;
  const int c0 = blk * a.bc, c1 = min(c0 + a.bc, nc);
  const int nchunks = c1 > c0 ? c1 - c0 : 0;
  float* dst = a.ws + ((size_t)(s * a.Hkv + g) * a.nb + blk) * K::E;
  if (nchunks == 0) {  // a block past the end of the sequence adds nothing
    for (int i = tid; i < K::E; i += kThreads) dst[i] = 0.0f;
    return;
  }
  uint8_t* sK = smem;       // stage st: K at st*KVT, V at st*KVT + KT
  uint8_t* sV = smem + K::KT;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + K::OFF_BAR);
  uint64_t* empty = full + K::NS;
  uint64_t* xf = empty + K::NS;
  uint64_t* s_full = xf + K::NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 2);
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < K::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&xf[i], 1);
    }
    mbar_init(s_full, 1);
    fence_mbar_init();
  }
  init_ones_block(smem + K::OFF_ONES, tid, kThreads);
  fence_proxy_async_smem();
  if (warp == 9) tmem_alloc(tmem_slot, K::TM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_flag = &s_abort;

  if (warp == 8) {
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < nchunks && ok; ++i) {
        const int st = i % K::NS, c = c0 + i;
        ok = mbar_wait(&empty[st], ((i / K::NS) & 1) ^ 1, abort_flag, a.err, kWaitLimitNs);
        if (!ok) break;
        mbar_arrive_expect_tx(&full[st], K::KT + K::VT);
        for (int bx = 0; bx < D / 64; ++bx)
          tma_load_3d(sK + st * K::KVT + bx * kBox, &tm_k, &full[st], bx * 64, g,
                      t0 + c * kChunk);
        for (int bx = 0; bx < DV / 64; ++bx)
          tma_load_3d(sV + st * K::KVT + bx * kBox, &tm_v, &full[st], bx * 64, g,
                      t0 + c * kChunk);
        ++issued;
      }
      if (!ok) {
        int dummy = 0;
        for (int i = (issued > K::NS ? issued - K::NS : 0); i < issued; ++i)
          mbar_wait(&full[i % K::NS], (i / K::NS) & 1, &dummy, nullptr, kWaitLimitNs);
      }
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // dv = 64: [V | 1] is one N = 80 MN-major operand whose second group is
      // the shared ones block (per-stage leading byte offset); dv = 128: the
      // ones column is a separate N = 16 product.
      constexpr uint32_t ID_SV = idesc_bf16_f32(D, DV == 64 ? DV + 16 : DV, 1, 1);
      constexpr uint32_t ID_S1 = idesc_bf16_f32(D, 16, 1, 1);
      const uint64_t dK = smem_desc_sw128(smem_u32(sK), kBox, 1024);
      const uint32_t ones = smem_u32(smem + K::OFF_ONES);
      const uint64_t d1 = smem_desc_sw128(ones, kBox, 1024);
      bool ok = true;
      for (int i = 0; i < nchunks && ok; ++i) {
        const int st = i % K::NS;
        ok = mbar_wait(&xf[st], (i / K::NS) & 1, abort_flag, a.err, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after();
        const uint32_t va = smem_u32(sV) + st * K::KVT;
        const uint64_t kd = desc_advance(dK, st * K::KVT);
        const uint64_t vd = smem_desc_sw128(va, DV == 64 ? ones - va : kBox, 1024);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          umma_f16_ss(tmem, desc_advance(kd, kk * 2048), desc_advance(vd, kk * 2048), ID_SV,
                      acc);
          if (DV != 64)
            umma_f16_ss(tmem + DV, desc_advance(kd, kk * 2048), desc_advance(d1, kk * 2048),
                        ID_S1, acc);
        }
        umma_commit(&empty[st]);
      }
      umma_commit(s_full);
      int dummy = 0;  // drain the tensor pipe before TMEM is released
      mbar_wait(s_full, 0, &dummy, nullptr, kWaitLimitNs);
    }
  } else {
    const int x = tid;
    bool ok = true;
    for (int i = 0; i < nchunks && ok; ++i) {
      const int st = i % K::NS, c = c0 + i;
      ok = mbar_wait(&full[st], (i / K::NS) & 1, abort_flag, a.err, kWaitLimitNs);
      if (!ok) break;
      const int valid = min(kChunk, ntok - c * kChunk);
      prep_tile<D / 64, kXf, VAR>(sK + st * K::KVT, valid, true, x);
      if (valid < kChunk || VAR::kIn != kInBf16)
        xf_tile<DV / 64, kXf, VAR>(sV + st * K::KVT, valid, false, x);
      fence_proxy_async_smem();
      named_bar_sync(1, kXf);
      if (x == 0) mbar_arrive(&xf[st]);
    }
    // store A_b.  M = 64 accumulator: state row 16*w + l in lane l < 16 of
    // sub-partition w; M = 128: row 32*w + l in lane l.
    if (ok && warp < 4) ok = mbar_wait(s_full, 0, abort_flag, a.err, kWaitLimitNs);
    if (ok && warp < 4) {
      tc_fence_after();
      const uint32_t t = tmem + ((uint32_t)(warp * 32) << 16);
      const bool has_row = (D == 128) || lane < 16;
      const int row = (D == 128) ? warp * 32 + lane : warp * 16 + lane;
#pragma unroll 1
      for (int cb = 0; cb < DV / 32; ++cb) {
        float v[32];
        tmem_ld32(t + cb * 32, v);
        tmem_wait_ld();
        if (has_row) {
          float4* d4 = reinterpret_cast<float4*>(dst + (size_t)row * DV + cb * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
      float zz[16];
      tmem_ld16(t + DV, zz);
      tmem_wait_ld();
      if (has_row) dst[D * DV + row] = zz[0];
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, K::TM_COLS);
  }
}

template <int D, int DV, class VAR = VarDefault>
cudaError_t launch(const FwdLaunch& p, int nb, int nblocks_launch, float* ws,
                   cudaStream_t stream) {
  using K = SCfg<D, DV>;
  CUtensorMap tk, tv;
  const bool f16 = VAR::kIn == kInF16;
  if (!make_tmap_3d(&tk, p.k, D, p.Hkv, p.total_tokens, 64, f16) ||
      !make_tmap_3d(&tv, p.v, DV, p.Hkv, p.total_tokens, 64, f16))
    return cudaErrorInvalidValue;
  StateArgs a;
  a.cu_seqlens = p.cu_seqlens;
  a.ws = ws;
  a.Hkv = p.Hkv;
  a.N = p.N;
  a.nb = nb;
  a.bc = block_chunks(p, nb);
  a.total_tokens = (int)p.total_tokens;
  a.err = p.err;
  auto kern = lt_block_state_kernel<D, DV, VAR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<dim3(nblocks_launch, p.Hkv, p.B), kThreads, K::SMEM, stream>>>(tk, tv, a);
  return cudaGetLastError();
}

// the input type and feature map of p as a compile-time variant
template <int D, int DV>
cudaError_t launch_var(const FwdLaunch& p, int nb, int nl, float* ws, cudaStream_t stream) {
  switch (p.in_f16 * 4 + p.phi) {
    case 0: return launch<D, DV, Var<kInBf16, kPhiElu1>>(p, nb, nl, ws, stream);
    case 1: return launch<D, DV, Var<kInBf16, kPhiRelu>>(p, nb, nl, ws, stream);
    case 2: return launch<D, DV, Var<kInBf16, kPhiExp>>(p, nb, nl, ws, stream);
    case 4: return launch<D, DV, Var<kInF16, kPhiElu1>>(p, nb, nl, ws, stream);
    case 5: return launch<D, DV, Var<kInF16, kPhiRelu>>(p, nb, nl, ws, stream);
    case 6: return launch<D, DV, Var<kInF16, kPhiExp>>(p, nb, nl, ws, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

// Blocks per sequence: enough CTAs to cover the SMs about once.  Packed
// sequences keep one block each (the sequences themselves give the
// parallelism).  lt_debug_set_schedule can force a count (tests, ablations).
int block_count(const FwdLaunch& p, int num_sms) {
  if (p.cu_seqlens) return 1;
  const int nc = (p.N + kChunk - 1) / kChunk;
  const int f = sched_blocks();
  if (f > 0) return f > nc ? nc : f;
  const int lanes = p.B * p.Hkv;
  int nb = num_sms / (lanes > 0 ? lanes : 1);
  if (nb < 1) nb = 1;
  if (nb > nc) nb = nc;
  const int bc = (nc + nb - 1) / nb;
  return (nc + bc - 1) / bc;  // no block left empty by the rounding
}

int block_chunks(const FwdLaunch& p, int nb) {
  if (nb <= 1) return 1 << 30;
  const int nc = (p.N + kChunk - 1) / kChunk;
  return (nc + nb - 1) / nb;
}

size_t block_workspace_bytes(const FwdLaunch& p, int nb) {
  return nb > 1 ? (size_t)p.B * p.Hkv * nb * (p.d * p.dv + p.d) * sizeof(float) : 0;
}

cudaError_t launch_block_state(const FwdLaunch& p, int nb, float* ws, cudaStream_t stream) {
  // causal: the last block's aggregate is never needed
  const int nl = p.causal ? nb - 1 : nb;
  if (nl <= 0) return cudaSuccess;
  if (p.in_f16 || p.phi) {  // variants: d = dv = 64 or 128
    if (p.d == 64 && p.dv == 64) return launch_var<64, 64>(p, nb, nl, ws, stream);
    if (p.d == 128 && p.dv == 128) return launch_var<128, 128>(p, nb, nl, ws, stream);
    return cudaErrorInvalidValue;
  }
  if (p.d == 64 && p.dv == 64) return launch<64, 64>(p, nb, nl, ws, stream);
  if (p.d == 128 && p.dv == 128) return launch<128, 128>(p, nb, nl, ws, stream);
  if (p.d == 64 && p.dv == 128) return launch<64, 128>(p, nb, nl, ws, stream);
  if (p.d == 128 && p.dv == 64) return launch<128, 64>(p, nb, nl, ws, stream);
  return cudaErrorInvalidValue;
}

}  // namespace lt
