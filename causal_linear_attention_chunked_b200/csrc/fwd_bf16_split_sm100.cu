// fwd_bf16_split_sm100.cu -- chunked linear attention (bf16 I/O, fp32
// accumulation) with one sequence split over a thread-block cluster.
//
// Same method as the sequential kernel (lineartile 1.0.0, "How It Works"
// and "Reference"; chunked evaluation with an inter-chunk carry as in "Why
// Stream Wins at Ultra-Long Context", section 5.3, whose two-level scan is
// what this kernel does across the CTAs of a cluster):
//     num_c = mask(phi(Q_c) phi(K_c)^T) [V_c|1] + phi(Q_c) [S|z]_<c
//     [S|z]_<c = sum_{c' < c} phi(K_c')^T [V_c'|1]
// A cluster of n CTAs owns one (sequence, KV head).  In round r, CTA i of
// the cluster takes chunk c = r*n + i.  Every round each CTA computes its
// chunk's state contribution dS_c = phi(K_c)^T [V_c|1] on the tensor cores
// (fp32 in TMEM) and the cluster forms the exclusive prefix over the round's
// n chunks through distributed shared memory, in two pushes: CTA j owns
// slice j of the d x (dv+1) state and keeps the running total of all
// earlier rounds for that slice in registers; every CTA sends each slice of
// its dS to the slice's owner, and each owner sends every CTA's exclusive
// prefix for its slice back to that CTA.  Both hops are bulk copies of the
// TMA engine between the CTAs' shared memories that complete transaction
// bytes on the receiver's mbarrier, so data and signal travel together.
// The score tile stays in TMEM: it is masked and rounded to bf16 in place
// and read back by the tensor cores as the A operand of P [V|1].
// The exchange for round r+1 runs while round r's score and output MMAs
// execute (the state MMA is issued one round ahead).  With n = 1 the state
// stays in the registers of the state warpgroup.
//
// Warp roles (448 threads):
//   warps 0-3   transform: phi in place on K and Q tiles, tail rows zeroed;
//               causal mask of the score tile, bf16 in place in TMEM
//   warps 4-7   epilogue: accumulator -> normalised bf16 rows -> global
//   warps 8-11  state: dS (TMEM) -> cluster exchange -> [S|z]_<c operand
//   warp 12     TMA producer
//   warp 13     TMEM allocator and single-thread MMA issuer
// d = dv = 64.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <mutex>

#include "fwd_common.cuh"
#include "lt_internal.h"
#include "lt_ptx.cuh"

namespace lt {
namespace {
using namespace fwd;

constexpr int D = 64, DV = 64;
constexpr int kThreads = 448;
constexpr int kMaxCluster = 16;
constexpr int kMaxClusterPad = 16;
constexpr int NQ = 4, NKV = 3;
constexpr int QT = kChunk * D * 2, KT = kChunk * D * 2, VT = kChunk * DV * 2;
constexpr int SOPT = (DV / 64 + 1) * D * kRowBytes;
constexpr int ZB = 2 * D * 4;              // z_c (column sums of phi(K_c)), 2 buffers
constexpr int CSB = 128 * 8 * 4;           // column-sum scratch of the transform warpgroup
constexpr int E = D * DV + D;  // state elements exchanged: S (row-major) then z
constexpr int E4 = E / 4;
constexpr int SLOT = E * 4;
constexpr int SLOT_IN = (E4 + kMaxClusterPad) * 16;  // n slices of <= ceil(E4/n) float4
constexpr int ZBASE = D * DV / 4;  // float4 index of the z block
constexpr int ACCW = DV + 16;
constexpr int TM_P = 0, TM_ACC = kChunk, TM_DS = TM_ACC + 2 * ACCW, TM_COLS = 512;
static_assert(TM_DS + 2 * ACCW <= TM_COLS, "TMEM budget");
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + NQ * QT;
constexpr int OFF_V = OFF_K + NKV * KT;
constexpr int OFF_SOP = OFF_V + NKV * VT;
constexpr int OFF_Z = OFF_SOP + SOPT;
constexpr int OFF_CS = OFF_Z + ZB;
constexpr int OFF_DS = OFF_CS + CSB;
constexpr int OFF_X = OFF_DS + SLOT_IN;
constexpr int OFF_BAR = OFF_X + SLOT;
constexpr int NBARS = 3 * NQ + 3 * NKV + 2 + 2 + 2 * 2 + 2 * 2 + 2 * 2 + 2 + 1;
constexpr int SMEM = OFF_BAR + NBARS * 8 + 16 + 1024;
static_assert(SMEM <= 232448, "shared memory budget");
constexpr int kMaxSliceIters = (E4 + 2 * 128 - 1) / (2 * 128);  // per thread, n >= 2

struct SBars {
  uint64_t *q_full, *q_empty, *q_xf, *kv_full, *kv_empty, *kv_xf;
  uint64_t *p_full, *pb_full, *sop_full, *sop_empty;
  uint64_t *ds_full, *ds_empty, *acc_full, *acc_empty, *z_full, *z_empty, *ds_in, *x_in, *drain;
};

__device__ __forceinline__ SBars carve(uint8_t* base) {
  uint64_t* b = reinterpret_cast<uint64_t*>(base);
  SBars r;
  r.q_full = b; b += NQ;
  r.q_empty = b; b += NQ;
  r.q_xf = b; b += NQ;
  r.kv_full = b; b += NKV;
  r.kv_empty = b; b += NKV;
  r.kv_xf = b; b += NKV;
  r.p_full = b++;
  r.pb_full = b++;
  r.sop_full = b++; r.sop_empty = b++;
  r.ds_full = b; b += 2;
  r.ds_empty = b; b += 2;
  r.acc_full = b; b += 2;
  r.acc_empty = b; b += 2;
  r.z_full = b; b += 2;
  r.z_empty = b; b += 2;
  r.ds_in = b++; r.x_in = b++;
  r.drain = b++;
  return r;
}

// Write one row of the [S | z 0 ... 0] operand (MN-major, 128-byte swizzle;
// row = state row a, columns n = 0..dv+15) from fp32 values (dv S entries
// and z).
__device__ __forceinline__ void write_sop_row(uint8_t* sop, int a, const float* s, float z) {
#pragma unroll
  for (int q8 = 0; q8 < DV / 8; ++q8) {
    const uint4 w = make_uint4(pack_bf16x2(s[q8 * 8 + 0], s[q8 * 8 + 1]),
                               pack_bf16x2(s[q8 * 8 + 2], s[q8 * 8 + 3]),
                               pack_bf16x2(s[q8 * 8 + 4], s[q8 * 8 + 5]),
                               pack_bf16x2(s[q8 * 8 + 6], s[q8 * 8 + 7]));
    *reinterpret_cast<uint4*>(sop + (q8 >> 3) * (D * kRowBytes) + sw128_off(a, q8 & 7)) = w;
  }
  const int grp = DV / 64;
  *reinterpret_cast<uint4*>(sop + grp * (D * kRowBytes) + sw128_off(a, 0)) =
      make_uint4(pack_bf16x2(z, 0.0f), 0u, 0u, 0u);
  *reinterpret_cast<uint4*>(sop + grp * (D * kRowBytes) + sw128_off(a, 1)) =
      make_uint4(0u, 0u, 0u, 0u);
}

// phi in place over the K tile (d = 64: one 128-byte-swizzled box; rows
// >= valid zeroed) and per-thread partial column sums of the result.
// Thread t (of 128) owns 16-byte pieces t + 128 i: rows (t >> 3) + 16 i,
// physical piece t & 7, hence logical columns 8 * ((t & 7) ^ ((t >> 3) & 7))
// .. +7 in every row it visits.
__device__ __forceinline__ void xf_k_colsum(uint8_t* tile, int valid, int t, float (&cs)[8]) {
#pragma unroll
  for (int e = 0; e < 8; ++e) cs[e] = 0.0f;
#pragma unroll 4
  for (int i = 0; i < kChunk * 8 / 128; ++i) {
    const int ch = t + 128 * i;
    uint4* p = reinterpret_cast<uint4*>(tile + ch * 16);
    uint4 v = *p;
    if ((ch >> 3) >= valid) {
      v = make_uint4(0u, 0u, 0u, 0u);
    } else {
      v.x = phi_bf16x2(v.x);
      v.y = phi_bf16x2(v.y);
      v.z = phi_bf16x2(v.z);
      v.w = phi_bf16x2(v.w);
    }
    *p = v;
    const float2 f0 = unpack_bf16x2(v.x), f1 = unpack_bf16x2(v.y);
    const float2 f2 = unpack_bf16x2(v.z), f3 = unpack_bf16x2(v.w);
    cs[0] += f0.x; cs[1] += f0.y; cs[2] += f1.x; cs[3] += f1.y;
    cs[4] += f2.x; cs[5] += f2.y; cs[6] += f3.x; cs[7] += f3.y;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    lt_fwd_split_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const FwdArgs a, const int ncl) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ci = (ncl > 1) ? (int)cluster_ctarank() : 0;  // rank in the cluster
  const int g = blockIdx.x / ncl;                           // KV head
  const int s = blockIdx.y;                                 // sequence
  int t0, ntok;
  if (a.cu_seqlens) {
    const int lo = a.cu_seqlens[s], hi = a.cu_seqlens[s + 1];
    if (lo < 0 || hi < lo || hi > a.total_tokens) {
      if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
      return;  // uniform over the cluster: every CTA reads the same bounds
    }
    t0 = lo;
    ntok = hi - lo;
  } else {
    t0 = s * a.N;
    ntok = a.N;
  }
  if (ntok <= 0) return;
  const int nc = (ntok + kChunk - 1) / kChunk;
  const int R = (nc + ncl - 1) / ncl;                        // rounds (whole cluster)
  const int Ri = ci < nc ? (nc - ci + ncl - 1) / ncl : 0;   // rounds with a chunk here
  const int G = a.G;

  uint8_t* sQ = smem + OFF_Q;
  uint8_t* sK = smem + OFF_K;
  uint8_t* sV = smem + OFF_V;
  uint8_t* sSOP = smem + OFF_SOP;
  float* sZ = reinterpret_cast<float*>(smem + OFF_Z);
  float* sCS = reinterpret_cast<float*>(smem + OFF_CS);
  float* sDSIN = reinterpret_cast<float*>(smem + OFF_DS);
  float* sX = reinterpret_cast<float*>(smem + OFF_X);
  SBars bars = carve(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + NBARS * 8);

  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&bars.q_full[i], 1);
      mbar_init(&bars.q_empty[i], 1);
      mbar_init(&bars.q_xf[i], 1);
    }
    for (int i = 0; i < NKV; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
      mbar_init(&bars.kv_xf[i], 1);
    }
    mbar_init(bars.p_full, 1);
    mbar_init(bars.pb_full, 1);
    mbar_init(bars.sop_full, 1);
    mbar_init(bars.sop_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.ds_full[i], 1);
      mbar_init(&bars.ds_empty[i], 1);
      mbar_init(&bars.acc_full[i], 1);
      mbar_init(&bars.acc_empty[i], 1);
      mbar_init(&bars.z_full[i], 1);
      mbar_init(&bars.z_empty[i], 1);
    }
    mbar_init(bars.ds_in, 1);
    mbar_init(bars.x_in, 1);
    mbar_init(bars.drain, 1);
    fence_mbar_init();
  }
  if (warp == 13) tmem_alloc(tmem_slot, TM_COLS);
  tc_fence_before();
  if (ncl > 1) cluster_sync_all(); else __syncthreads();  // peers' barriers are initialised
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_flag = &s_abort;
  const bool causal = a.causal != 0;
  const int n_items = Ri * G;

  if (warp == 12) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && Ri > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int q_issued = 0, kv_issued = 0;
      bool ok = true;
      auto load_kv = [&](int r) -> bool {
        const int st = r % NKV, c = r * ncl + ci;
        if (!mbar_wait(&bars.kv_empty[st], ((r / NKV) & 1) ^ 1, abort_flag, a.err, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars.kv_full[st], KT + VT);
        tma_load_3d(sK + st * KT, &tm_k, &bars.kv_full[st], 0, g, t0 + c * kChunk);
        tma_load_3d(sV + st * VT, &tm_v, &bars.kv_full[st], 0, g, t0 + c * kChunk);
        ++kv_issued;
        return true;
      };
      auto load_q = [&](int j) -> bool {
        const int st = j % NQ, r = j / G, h = j % G, c = r * ncl + ci;
        if (!mbar_wait(&bars.q_empty[st], ((j / NQ) & 1) ^ 1, abort_flag, a.err, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars.q_full[st], QT);
        tma_load_3d(sQ + st * QT, &tm_q, &bars.q_full[st], 0, g * G + h, t0 + c * kChunk);
        ++q_issued;
        return true;
      };
      if (causal) {
        for (int r = 0; r < Ri && ok; ++r) {
          ok = load_kv(r);
          for (int h = 0; h < G && ok; ++h) ok = load_q(r * G + h);
        }
      } else {
        for (int r = 0; r < Ri && ok; ++r) ok = load_kv(r);
        for (int j = 0; j < n_items && ok; ++j) ok = load_q(j);
      }
      if (!ok) {  // drain copies in flight (bounded, ignoring the abort flag)
        int dummy = 0;
        for (int r = (kv_issued > NKV ? kv_issued - NKV : 0); r < kv_issued; ++r)
          mbar_wait(&bars.kv_full[r % NKV], (r / NKV) & 1, &dummy, nullptr, kWaitLimitNs);
        for (int j = (q_issued > NQ ? q_issued - NQ : 0); j < q_issued; ++j)
          mbar_wait(&bars.q_full[j % NQ], (j / NQ) & 1, &dummy, nullptr, kWaitLimitNs);
      }
    }
  } else if (warp == 13) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_P = idesc_bf16_f32(kChunk, kChunk, 0, 0);
      constexpr uint32_t ID_SV = idesc_bf16_f32(D, DV + 0, 1, 1);
      constexpr uint32_t ID_PV = idesc_bf16_f32(kChunk, DV, 0, 1);
      constexpr uint32_t ID_QS = idesc_bf16_f32(kChunk, DV + 16, 0, 1);
      // descriptor bases, advanced per stage / K step with one 64-bit add
      const uint64_t dQk = smem_desc_sw128(smem_u32(sQ), 16, 1024);      // K-major
      const uint64_t dKk = smem_desc_sw128(smem_u32(sK), 16, 1024);      // K-major
      const uint64_t dKmn = smem_desc_sw128(smem_u32(sK), kBox, 1024);   // MN-major
      const uint64_t dVmn = smem_desc_sw128(smem_u32(sV), kBox, 1024);   // MN-major
      const uint64_t dSop = smem_desc_sw128(smem_u32(sSOP), D * kRowBytes, 1024);
      bool ok = true;
      // dS (or the running S for non-causal) = phi(K)^T V
      auto issue_ds = [&](int r, uint32_t t_ds, bool accumulate) {
        const int st = r % NKV;
        const uint64_t ka = desc_advance(dKmn, st * KT), vb = desc_advance(dVmn, st * VT);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          umma_f16_ss(t_ds, desc_advance(ka, kk * 2048), desc_advance(vb, kk * 2048), ID_SV,
                      (accumulate || kk > 0) ? 1u : 0u);
      };
      // Acc (+)= phi(Q) [S | z 0 ..]
      auto issue_qs = [&](uint32_t t_acc, int qs, bool accumulate) {
        const uint64_t qa = desc_advance(dQk, qs * QT);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_f16_ss(t_acc, desc_advance(qa, (kk >> 2) * kBox + (kk & 3) * 32),
                      desc_advance(dSop, kk * 2048), ID_QS, (accumulate || kk > 0) ? 1u : 0u);
      };
      if (causal) {
        auto state_mma = [&](int r) -> bool {
          const int b = r & 1;
          if (!mbar_wait(&bars.kv_xf[r % NKV], (r / NKV) & 1, abort_flag, a.err, kWaitLimitNs) ||
              !mbar_wait(&bars.ds_empty[b], ((r >> 1) & 1) ^ 1, abort_flag, a.err, kWaitLimitNs))
            return false;
          tc_fence_after();
          issue_ds(r, tmem + TM_DS + b * ACCW, false);
          umma_commit(&bars.ds_full[b]);
          return true;
        };
        if (Ri > 0) ok = state_mma(0);
        for (int r = 0; r < Ri && ok; ++r) {
          const uint64_t kd = desc_advance(dKk, (r % NKV) * KT);
          const uint64_t vd = desc_advance(dVmn, (r % NKV) * VT);
          for (int h = 0; h < G && ok; ++h) {
            const int j = r * G + h, qs = j % NQ, as = j & 1;
            const uint64_t qd = desc_advance(dQk, qs * QT);
            const uint32_t t_acc = tmem + TM_ACC + as * ACCW;
            // The score tile of the previous item was read by its P [V|1]
            // MMAs, issued before this one: the tensor pipe runs them in order.
            ok = mbar_wait(&bars.q_xf[qs], (j / NQ) & 1, abort_flag, a.err, kWaitLimitNs);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t o = (kk >> 2) * kBox + (kk & 3) * 32;
              umma_f16_ss(tmem + TM_P, desc_advance(qd, o), desc_advance(kd, o), ID_P,
                          kk > 0 ? 1u : 0u);
            }
            umma_commit(bars.p_full);
            // the next round's state MMA (its exchange then overlaps this
            // round's work), issued after the score MMA so that the score
            // tile does not wait for the next K tile
            if (h == 0 && r + 1 < Ri) {
              ok = state_mma(r + 1);
              if (!ok) break;
            }
            ok = mbar_wait(bars.pb_full, j & 1, abort_flag, a.err, kWaitLimitNs) &&
                 mbar_wait(&bars.acc_empty[as], ((j >> 1) & 1) ^ 1, abort_flag, a.err,
                           kWaitLimitNs);
            if (!ok) break;
            tc_fence_after();
            // P V: bf16 scores from TMEM, 16 keys (8 columns) per MMA.  The
            // normaliser column of the accumulator was initialised with the
            // score row sums by the transform warpgroup.
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk)
              umma_f16_ts(t_acc, tmem + TM_P + kk * 8, desc_advance(vd, kk * 2048), ID_PV,
                          kk > 0 ? 1u : 0u);
            if (h == G - 1) umma_commit(&bars.kv_empty[r % NKV]);
            if (h == 0) {
              ok = mbar_wait(bars.sop_full, r & 1, abort_flag, a.err, kWaitLimitNs);
              if (!ok) break;
              tc_fence_after();
            }
            issue_qs(t_acc, qs, true);
            umma_commit(&bars.acc_full[as]);
            umma_commit(&bars.q_empty[qs]);
          }
          if (ok) umma_commit(bars.sop_empty);
        }
      } else {
        for (int r = 0; r < Ri && ok; ++r) {
          ok = mbar_wait(&bars.kv_xf[r % NKV], (r / NKV) & 1, abort_flag, a.err, kWaitLimitNs);
          if (!ok) break;
          tc_fence_after();
          issue_ds(r, tmem + TM_DS, r > 0);
          umma_commit(&bars.kv_empty[r % NKV]);
        }
        if (ok) umma_commit(&bars.ds_full[0]);
        if (ok && n_items > 0) ok = mbar_wait(bars.sop_full, 0, abort_flag, a.err, kWaitLimitNs);
        for (int j = 0; j < n_items && ok; ++j) {
          const int qs = j % NQ, as = j & 1;
          ok = mbar_wait(&bars.q_xf[qs], (j / NQ) & 1, abort_flag, a.err, kWaitLimitNs) &&
               mbar_wait(&bars.acc_empty[as], ((j >> 1) & 1) ^ 1, abort_flag, a.err,
                         kWaitLimitNs);
          if (!ok) break;
          tc_fence_after();
          issue_qs(tmem + TM_ACC + as * ACCW, qs, false);
          umma_commit(&bars.acc_full[as]);
          umma_commit(&bars.q_empty[qs]);
        }
      }
      umma_commit(bars.drain);
      int dummy = 0;
      mbar_wait(bars.drain, 0, &dummy, nullptr, kWaitLimitNs);
    }
  } else if (warp < 4) {
    // ----------------------------------------------- transform warpgroup
    const int x = tid;
    bool ok = true;
    // z of the chunk (column sums of phi(K_c)) -> sZ[r & 1] (causal), or a
    // running total over this CTA's chunks (non-causal, published once).
    float zrun = 0.0f;
    auto xf_kv = [&](int r) -> bool {
      const int st = r % NKV, c = r * ncl + ci;
      if (!mbar_wait(&bars.kv_full[st], (r / NKV) & 1, abort_flag, a.err, kWaitLimitNs))
        return false;
      const int valid = min(kChunk, ntok - c * kChunk);
      float cs[8];
      xf_k_colsum(sK + st * KT, valid, x, cs);
      if (valid < kChunk) xf_tile<DV / 64>(sV + st * VT, valid, false, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) sCS[x * 8 + e] = cs[e];
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (x == 0) mbar_arrive(&bars.kv_xf[st]);
      float zc = 0.0f;
      if (x < D) {  // column x: logical piece x/8 is held by 16 threads
        const int jj = x >> 3, e = x & 7;
#pragma unroll
        for (int rg = 0; rg < 16; ++rg) zc += sCS[(8 * rg + (jj ^ (rg & 7))) * 8 + e];
      }
      if (causal) {
        const int b = r & 1;
        if (!mbar_wait(&bars.z_empty[b], ((r >> 1) & 1) ^ 1, abort_flag, a.err, kWaitLimitNs))
          return false;
        if (x < D) sZ[b * D + x] = zc;
        named_bar_sync(1, 128);
        if (x == 0) mbar_arrive(&bars.z_full[b]);
      } else {
        zrun += zc;
        named_bar_sync(1, 128);  // the scratch is rewritten by the next tile
      }
      return true;
    };
    auto xf_q = [&](int j) -> bool {
      const int st = j % NQ;
      if (!mbar_wait(&bars.q_full[st], (j / NQ) & 1, abort_flag, a.err, kWaitLimitNs))
        return false;
      xf_tile<D / 64>(sQ + st * QT, kChunk, true, x);
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (x == 0) mbar_arrive(&bars.q_xf[st]);
      return true;
    };
    // causal mask of the score tile and bf16 rounding, in place in TMEM:
    // fp32 columns [32b, 32b+32) become packed bf16 columns [16b, 16b+16),
    // which only overwrites columns this thread has already read
    auto mask_p = [&](int j) -> bool {
      const int as = j & 1;
      if (!mbar_wait(bars.p_full, j & 1, abort_flag, a.err, kWaitLimitNs) ||
          !mbar_wait(&bars.acc_empty[as], ((j >> 1) & 1) ^ 1, abort_flag, a.err, kWaitLimitNs))
        return false;
      tc_fence_after();
      const uint32_t lane_sel = (uint32_t)(warp * 32) << 16;
      const uint32_t t_p = tmem + TM_P + lane_sel;
      const int row = x;
      float rs = 0.0f;  // row sum of the rounded, masked scores
#pragma unroll
      for (int b = 0; b < kChunk / 32; ++b) {
        uint32_t pk[16];
        if (b <= warp) {  // warp-uniform: blocks right of the diagonal are all zero
          float r[32];
          tmem_ld32(t_p + b * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float lo = (b * 32 + 2 * e > row) ? 0.0f : r[2 * e];
            const float hi = (b * 32 + 2 * e + 1 > row) ? 0.0f : r[2 * e + 1];
            pk[e] = pack_bf16x2(lo, hi);
            const float2 rr = unpack_bf16x2(pk[e]);
            rs += rr.x + rr.y;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        }
        tmem_st16(t_p + b * 16, pk);
      }
      // the normaliser column of this item's accumulator starts at the row
      // sum; the phi(Q) [S|z] MMA accumulates phi(Q) z onto it
      tmem_st1(tmem + TM_ACC + as * ACCW + DV + lane_sel, __float_as_uint(rs));
      tmem_wait_st();
      tc_fence_before();
      named_bar_sync(1, 128);
      if (x == 0) mbar_arrive(bars.pb_full);
      return true;
    };
    if (causal) {
      if (Ri > 0) ok = xf_kv(0);
      for (int r = 0; r < Ri && ok; ++r) {
        for (int h = 0; h < G && ok; ++h) {
          ok = xf_q(r * G + h);
          // next K tile while this round's score MMA runs
          if (ok && h == 0 && r + 1 < Ri) ok = xf_kv(r + 1);
          if (ok) ok = mask_p(r * G + h);
        }
      }
    } else {
      for (int r = 0; r < Ri && ok; ++r) ok = xf_kv(r);
      if (ok) {  // this CTA's z total (zero when it has no chunk)
        if (x < D) sZ[x] = zrun;
        named_bar_sync(1, 128);
        if (x == 0) mbar_arrive(&bars.z_full[0]);
      }
      for (int j = 0; j < n_items && ok; ++j) ok = xf_q(j);
    }
  } else if (warp < 8) {
    // ----------------------------------------------- epilogue warpgroup
    const int x = tid - 128, sp = warp & 3;
    const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
    bool ok = true;
    for (int j = 0; j < n_items && ok; ++j) {
      const int r = j / G, h = j % G, as = j & 1, c = r * ncl + ci;
      ok = mbar_wait(&bars.acc_full[as], (j >> 1) & 1, abort_flag, a.err, kWaitLimitNs);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_acc = tmem + TM_ACC + as * ACCW + lane_base;
      float den[16], n0[32], n1[32];
      tmem_ld16(t_acc + DV, den);
      tmem_ld32(t_acc, n0);
      tmem_ld32(t_acc + 32, n1);
      tmem_wait_ld();
      tc_fence_before();
      named_bar_sync(2, 128);
      if (x == 0) mbar_arrive(&bars.acc_empty[as]);
      const float inv = 1.0f / (den[0] + a.eps);
      const int valid = min(kChunk, ntok - c * kChunk);
      if (x < valid) {
        __nv_bfloat16* orow =
            a.out + ((size_t)(t0 + c * kChunk + x) * a.Hq + (size_t)(g * G + h)) * DV;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          *reinterpret_cast<uint4*>(orow + q4 * 8) =
              make_uint4(pack_bf16x2(n0[q4 * 8 + 0] * inv, n0[q4 * 8 + 1] * inv),
                         pack_bf16x2(n0[q4 * 8 + 2] * inv, n0[q4 * 8 + 3] * inv),
                         pack_bf16x2(n0[q4 * 8 + 4] * inv, n0[q4 * 8 + 5] * inv),
                         pack_bf16x2(n0[q4 * 8 + 6] * inv, n0[q4 * 8 + 7] * inv));
          *reinterpret_cast<uint4*>(orow + 32 + q4 * 8) =
              make_uint4(pack_bf16x2(n1[q4 * 8 + 0] * inv, n1[q4 * 8 + 1] * inv),
                         pack_bf16x2(n1[q4 * 8 + 2] * inv, n1[q4 * 8 + 3] * inv),
                         pack_bf16x2(n1[q4 * 8 + 4] * inv, n1[q4 * 8 + 5] * inv),
                         pack_bf16x2(n1[q4 * 8 + 6] * inv, n1[q4 * 8 + 7] * inv));
        }
      }
    }
  } else if (warp < 12) {
    // -------------------------------------------------- state warpgroup
    // dS is an M=64 accumulator: state row a = 16*sp + l lives in lane l < 16
    // of TMEM sub-partition sp.  State layout in float4 units: row a of S is
    // [16a, 16a+16), z[a] is component a%4 of float4 1024 + a/4.
    const int y = tid - 256, sp = warp & 3;
    const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
    const bool has_row = lane < 16;
    const int row = sp * 16 + lane;
    bool ok = true;
    auto publish_sop = [&](int r, const float* sv, float z) -> bool {
      if (!mbar_wait(bars.sop_empty, (r & 1) ^ 1, abort_flag, a.err, kWaitLimitNs)) return false;
      if (has_row) write_sop_row(sSOP, row, sv, z);
      fence_proxy_async_smem();
      named_bar_sync(3, 128);
      if (y == 0) mbar_arrive(bars.sop_full);
      return true;
    };
    // State vector order (float4 units): S float4 q of row a at q*64 + a
    // (column-block major, so a warp's rows are contiguous: no bank
    // conflicts), z[a] is component a%4 of float4 ZBASE + a/4.
    // The prefix delivered for this thread's row, from the local X slot:
    auto x_row = [&](float* xs, float& xz) {
      if (has_row) {
        const float4* X4 = reinterpret_cast<const float4*>(sX);
#pragma unroll
        for (int q = 0; q < DV / 4; ++q) {
          const float4 t4 = X4[q * D + row];
          xs[4 * q] = t4.x;
          xs[4 * q + 1] = t4.y;
          xs[4 * q + 2] = t4.z;
          xs[4 * q + 3] = t4.w;
        }
        xz = sX[ZBASE * 4 + row];
      }
    };
    if (causal && ncl == 1) {
      // one CTA per sequence: the running state lives in registers
      float T[DV], Tz = 0.0f;
#pragma unroll
      for (int e = 0; e < DV; ++e) T[e] = 0.0f;
      for (int r = 0; r < Ri && ok; ++r) {
        ok = publish_sop(r, T, Tz);  // [S|z]_<c does not need this round's dS
        if (!ok) break;
        const int b = r & 1;
        ok = mbar_wait(&bars.ds_full[b], (r >> 1) & 1, abort_flag, a.err, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after();
        const uint32_t t = tmem + TM_DS + b * ACCW + lane_base;
#pragma unroll
        for (int half = 0; half < DV / 32; ++half) {
          float c0[32];
          tmem_ld32(t + half * 32, c0);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) T[half * 32 + e] += c0[e];
        }
        tc_fence_before();
        ok = mbar_wait(&bars.z_full[b], (r >> 1) & 1, abort_flag, a.err, kWaitLimitNs);
        if (!ok) break;
        if (has_row) Tz += sZ[b * D + row];
        named_bar_sync(3, 128);
        if (y == 0) {
          mbar_arrive(&bars.ds_empty[b]);
          mbar_arrive(&bars.z_empty[b]);
        }
      }
    } else {
      // Cluster exchange (causal: exclusive prefix per round; non-causal: one
      // all-reduce).  CTA o owns the float4 slice [lo(o), lo(o+1)) of the
      // state.  Hop 1: every CTA stages its dS in its X slot and sends slice
      // o to CTA o's receive slot (row ci).  Hop 2: the owner turns the n
      // received slices in place into the n exclusive prefixes and sends
      // slice j back into CTA j's X slot.  Both hops are TMA bulk copies
      // that complete transaction bytes on the receiver's mbarrier.
      const int SMAX = (E4 + ncl - 1) / ncl;
      const int lo = (ci * E4) / ncl, hi = ((ci + 1) * E4) / ncl, len = hi - lo;
      const uint32_t in_local = smem_u32(sDSIN), x_local = smem_u32(sX);
      const uint32_t in_bar = smem_u32(bars.ds_in), x_bar = smem_u32(bars.x_in);
      float4* X4 = reinterpret_cast<float4*>(sX);
      float4* IN4 = reinterpret_cast<float4*>(sDSIN);
      // this thread's dS row (TMEM buffer b, or zeros) -> X slot
      auto stage_ds = [&](int b, int zb, bool have) {
        const uint32_t t = tmem + TM_DS + b * ACCW + lane_base;
        float z = 0.0f;
#pragma unroll
        for (int half = 0; half < DV / 32; ++half) {
          float c0[32];
          if (have) {
            tmem_ld32(t + half * 32, c0);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) c0[e] = 0.0f;
          }
          if (has_row) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              X4[(half * 8 + q) * D + row] =
                  make_float4(c0[4 * q], c0[4 * q + 1], c0[4 * q + 2], c0[4 * q + 3]);
          }
        }
        if (have && has_row) z = sZ[zb * D + row];  // z_full[zb] already observed
        if (has_row) sX[ZBASE * 4 + row] = z;
      };
      auto expect_round = [&]() {
        if (y == 0) {
          mbar_arrive_expect_tx(bars.ds_in, (uint32_t)(ncl * len * 16));
          mbar_arrive_expect_tx(bars.x_in, (uint32_t)(E4 * 16));
        }
      };
      // hop 1 (after every staging write is done and proxy-fenced)
      auto send_slices = [&]() {
        if (y == 0) {
          for (int o = 0; o < ncl; ++o) {
            const int olo = (o * E4) / ncl, ohi = ((o + 1) * E4) / ncl;
            bulk_copy_to_cluster(mapa_shared(in_local, (uint32_t)o) + (uint32_t)(ci * SMAX) * 16u,
                                 x_local + (uint32_t)olo * 16u, (uint32_t)(ohi - olo) * 16u,
                                 mapa_shared(in_bar, (uint32_t)o));
          }
        }
      };
      // hop 2: receive-slot row j now holds CTA j's prefix of my slice
      auto return_slices = [&]() {
        if (y == 0) {
          for (int j = 0; j < ncl; ++j)
            bulk_copy_to_cluster(mapa_shared(x_local, (uint32_t)j) + (uint32_t)lo * 16u,
                                 in_local + (uint32_t)(j * SMAX) * 16u, (uint32_t)len * 16u,
                                 mapa_shared(x_bar, (uint32_t)j));
        }
      };
      if (causal) {
        float4 T[kMaxSliceIters];
#pragma unroll
        for (int k = 0; k < kMaxSliceIters; ++k) T[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < R && ok; ++r) {
          const bool active = r < Ri;
          expect_round();
          if (active) {
            const int b = r & 1;
            ok = mbar_wait(&bars.ds_full[b], (r >> 1) & 1, abort_flag, a.err, kWaitLimitNs) &&
                 mbar_wait(&bars.z_full[b], (r >> 1) & 1, abort_flag, a.err, kWaitLimitNs);
            if (!ok) break;
            tc_fence_after();
            stage_ds(b, b, true);
            tc_fence_before();
          } else {
            stage_ds(0, 0, false);
          }
          fence_proxy_async_smem();
          named_bar_sync(3, 128);
          if (active && y == 0) {
            mbar_arrive(&bars.ds_empty[r & 1]);
            mbar_arrive(&bars.z_empty[r & 1]);
          }
          send_slices();
          ok = mbar_wait_cluster(bars.ds_in, r & 1, abort_flag, a.err, kWaitLimitNs);
          if (!ok) break;
#pragma unroll
          for (int k = 0; k < kMaxSliceIters; ++k) {
            const int e = y + 128 * k;
            if (e < len) {
              float4 p = T[k];
              for (int j = 0; j < ncl; ++j) {
                const float4 vj = IN4[j * SMAX + e];
                IN4[j * SMAX + e] = p;
                p.x += vj.x;
                p.y += vj.y;
                p.z += vj.z;
                p.w += vj.w;
              }
              T[k] = p;
            }
          }
          fence_proxy_async_smem();
          named_bar_sync(3, 128);
          return_slices();
          ok = mbar_wait_cluster(bars.x_in, r & 1, abort_flag, a.err, kWaitLimitNs);
          if (!ok) break;
          if (active) {
            float xs[DV];
            float xz = 0.0f;
            x_row(xs, xz);
            ok = publish_sop(r, xs, xz);
          }
        }
      } else {
        expect_round();
        ok = mbar_wait(&bars.ds_full[0], 0, abort_flag, a.err, kWaitLimitNs) &&
             mbar_wait(&bars.z_full[0], 0, abort_flag, a.err, kWaitLimitNs);
        if (ok) {
          tc_fence_after();
          stage_ds(0, 0, Ri > 0);
          tc_fence_before();
          fence_proxy_async_smem();
          named_bar_sync(3, 128);
          send_slices();
          ok = mbar_wait_cluster(bars.ds_in, 0, abort_flag, a.err, kWaitLimitNs);
        }
        if (ok) {
          for (int e = y; e < len; e += 128) {
            float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < ncl; ++j) {
              const float4 vj = IN4[j * SMAX + e];
              p.x += vj.x;
              p.y += vj.y;
              p.z += vj.z;
              p.w += vj.w;
            }
            for (int j = 0; j < ncl; ++j) IN4[j * SMAX + e] = p;
          }
          fence_proxy_async_smem();
          named_bar_sync(3, 128);
          return_slices();
          ok = mbar_wait_cluster(bars.x_in, 0, abort_flag, a.err, kWaitLimitNs);
        }
        if (ok && Ri > 0) {
          float xs[DV];
          float xz = 0.0f;
          x_row(xs, xz);
          ok = publish_sop(0, xs, xz);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (ncl > 1) cluster_sync_all();  // no peer touches this CTA's shared memory any more
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// ------------------------------------------------------------- host side
int env_int(const char* name, int dflt) {
  const char* v = getenv(name);
  return v ? atoi(v) : dflt;
}

struct ClusterInfo {
  int max_active[kMaxCluster + 1];
  bool ready;
};
ClusterInfo g_info[64];
std::mutex g_info_mu;

// Number of clusters of each size that can be resident at once.
const ClusterInfo* cluster_info(int dev) {
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_info_mu);
  ClusterInfo& ci = g_info[dev];
  if (!ci.ready) {
    auto kern = lt_fwd_split_kernel;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    for (int n = 1; n <= kMaxCluster; ++n) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(n * 16, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = SMEM;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = n;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int num = 0;
      if (cudaOccupancyMaxActiveClusters(&num, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        num = 0;
      }
      ci.max_active[n] = num;
    }
    ci.ready = true;
  }
  return &ci;
}

// Cluster size: minimise (waves of clusters) x (rounds per CTA).
int choose_cluster(int lanes, int nc, int dev) {
  const int forced = env_int("LT_SPLIT_N", 0);
  if (forced >= 1 && forced <= kMaxCluster) return forced < nc ? forced : (nc > 0 ? nc : 1);
  const ClusterInfo* info = cluster_info(dev);
  if (!info) return 1;
  int best = 1;
  long long best_t = -1;
  for (int n = 1; n <= kMaxCluster && n <= nc; ++n) {
    const int act = info->max_active[n];
    if (act <= 0) continue;
    const long long waves = (lanes + act - 1) / act;
    const long long t = waves * ((nc + n - 1) / n);
    if (best_t < 0 || t < best_t) {
      best_t = t;
      best = n;
    }
  }
  return best;
}

}  // namespace

bool split_supported(const FwdLaunch& p) { return p.d == 64 && p.dv == 64; }

cudaError_t launch_fwd_bf16_split(const FwdLaunch& p, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (!make_tmap_3d(&tq, p.q, D, p.Hq, p.total_tokens, 64) ||
      !make_tmap_3d(&tk, p.k, D, p.Hkv, p.total_tokens, 64) ||
      !make_tmap_3d(&tv, p.v, DV, p.Hkv, p.total_tokens, 64))
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  auto kern = lt_fwd_split_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  // packed sequences have unequal lengths: one CTA per (sequence, KV head)
  const int nc = p.cu_seqlens ? 1 : (p.N + kChunk - 1) / kChunk;
  const int ncl = p.cu_seqlens ? 1 : choose_cluster(p.B * p.Hkv, nc, dev);
  FwdArgs a;
  a.ws = nullptr;
  a.nb = 1;
  a.bc = 1 << 30;
  a.out = reinterpret_cast<__nv_bfloat16*>(p.out);
  a.cu_seqlens = p.cu_seqlens;
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.N = p.N;
  a.G = p.Hq / p.Hkv;
  a.causal = p.causal;
  a.eps = p.eps;
  a.total_tokens = (int)p.total_tokens;
  a.err = p.err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ncl * p.Hkv, p.B, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = ncl;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, a, ncl);
  return e;
}

}  // namespace lt
