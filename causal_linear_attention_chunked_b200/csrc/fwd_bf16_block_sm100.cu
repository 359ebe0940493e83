// fwd_bf16_block_sm100.cu -- block-parallel chunked linear attention, bf16
// I/O with fp32 accumulation, for d = dv = 64 (sm_100a: tcgen05 + TMA + TMEM).
//
// Method (lineartile 1.0.0, "How It Works" and "Reference"):
//     O_i = phi(Q_i) S_i / (phi(Q_i) . z_i + eps),  S_i = sum_{j<=i} phi(K_j)^T V_j,
//     z_i = sum_{j<=i} phi(K_j),  phi(x) = ELU(x) + 1.
// Evaluation is the two-level chunked scan of "Why Stream Wins at
// Ultra-Long Context", section 5.3 (chunk-local work, an inter-chunk carry,
// and a broadcast correction), applied twice:
//   * a sequence is cut into blocks of Bc chunks of 128 tokens;
//   * lt_block_state_kernel: one CTA per block computes the block aggregate
//     A_b = sum_{c in b} phi(K_c)^T [V_c | 1]  (fp32, to a workspace);
//   * lt_block_fwd_kernel: one CTA per block walks its chunks in order,
//     starting from the carry sum_{b' < b} A_b' and then carrying
//     [S|z] += phi(K_c)^T [V_c|1] from chunk to chunk, and computes
//         num_c = mask(phi(Q_c) phi(K_c)^T) V_c + phi(Q_c) S_<c
//         den_c = mask(phi(Q_c) phi(K_c)^T) 1   + phi(Q_c) z_<c
//     on the tensor cores.
// No CTA waits on another: the two launches are ordered on the stream.
// With one block per sequence the first launch is skipped.
// Non-causal mode: the state kernel computes every block's sum and the
// forward kernel reads only Q, with [S|z] = sum of all blocks.
//
// Forward-kernel warp roles (576 threads; TMEM sub-partition = warp % 4):
//   warps 0-7   transform: phi in place on K and Q tiles (tail rows zeroed)
//   warps 8-11  mask + epilogue: causal mask of the score tile, bf16 in
//               place in TMEM; accumulator -> normalised bf16 rows -> global
//   warps 12-15 state: carry into the TMEM state accumulator, which the
//               tensor cores advance by phi(K)^T [V | 1] per chunk; TMEM
//               state -> bf16 B operand before every chunk
//   warp 16     TMA producer
//   warp 17     TMEM allocator and single-thread MMA issuer
// The normaliser is the extra column of P [V | 1] and phi(Q) [S | z].
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include "fwd_common.cuh"
#include "lt_internal.h"
#include "lt_state.h"
#include "lt_ptx.cuh"

namespace lt {
namespace {
using namespace fwd;

constexpr int D = 64, DV = 64;
constexpr int E = D * DV + D;  // block aggregate: S (row-major d x dv) then z
constexpr int QT = kChunk * D * 2, KT = kChunk * D * 2, VT = kChunk * DV * 2;
constexpr int KVT = KT + VT;  // one K/V stage: [K][V]
constexpr int SOPT = (DV / 64 + 1) * D * kRowBytes;
constexpr int ONEST = kChunk * kRowBytes;
constexpr int ACCW = DV + 16;

struct BlockArgs {
  __nv_bfloat16* out;
  const int32_t* cu_seqlens;
  float* ws;        // block aggregates [lane][nb][E], or nullptr
  int carry_pre;    // 1: slot b of ws already holds block b's carry (every block reads it)
  int Hq, Hkv, N, G, causal;
  int nb;           // blocks per sequence (lane)
  int bc;           // chunks per block
  float eps;
  int total_tokens;
  int* err;
};

__device__ __forceinline__ bool seq_bounds(const BlockArgs& a, int s, int& t0, int& n) {
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

// ========================================================================
// Forward pass over one block per CTA.
// ========================================================================
constexpr int kThreads = 576;
constexpr int kXf = 256;  // transform threads (warps 0-7, two per SM sub-partition)
constexpr int NQ = 4;
constexpr int OSTT = kChunk * DV * 2;  // one output staging tile
// two score tiles (item j uses j & 1), two accumulators, the running state
constexpr int TM_P = 0, TM_ACC = 2 * kChunk, TM_S = TM_ACC + 2 * ACCW, TM_COLS = 512;
static_assert(TM_S + ACCW <= TM_COLS, "TMEM budget");
// Shared-memory layout.  kTma (the TMA-store image) trades one of the four
// K/V stages for two output staging tiles.
template <bool kTma>
struct BL {
  static constexpr int NKV = kTma ? 3 : 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + NQ * QT;  // stage st: [K][V] at st*KVT
  static constexpr int OFF_ONES = OFF_KV + NKV * KVT;
  static constexpr int OFF_SOP = OFF_ONES + ONEST;
  static constexpr int OFF_Z = OFF_SOP + SOPT;
  static constexpr int OFF_OST = (OFF_Z + D * 4 + 1023) & ~1023;  // kTma: two staging tiles
  static constexpr int OFF_BAR = kTma ? OFF_OST + 2 * OSTT : OFF_Z + D * 4;
  static constexpr int NBARS = 3 * NQ + 3 * NKV + 2 * 2 + 2 + 2 + 2 * 2 + 1;
  static constexpr int SMEM = OFF_BAR + NBARS * 8 + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct Bars {
  uint64_t *q_full, *q_empty, *q_xf, *kv_full, *kv_empty, *kv_xf;
  uint64_t *p_full, *pb_full, *sop_full, *sop_empty;
  uint64_t *s_full, *s_empty, *acc_full, *acc_empty, *drain;
};

template <int NKV>
__device__ __forceinline__ Bars carve(uint8_t* base) {
  uint64_t* b = reinterpret_cast<uint64_t*>(base);
  Bars r;
  r.q_full = b; b += NQ;
  r.q_empty = b; b += NQ;
  r.q_xf = b; b += NQ;
  r.kv_full = b; b += NKV;
  r.kv_empty = b; b += NKV;
  r.kv_xf = b; b += NKV;
  r.p_full = b; b += 2;
  r.pb_full = b; b += 2;
  r.sop_full = b++;
  r.sop_empty = b++;
  r.s_full = b++;
  r.s_empty = b++;
  r.acc_full = b; b += 2;
  r.acc_empty = b; b += 2;
  r.drain = b++;
  return r;
}

// Sum, in block order, of the aggregates of blocks [0, nsum) of one lane
// (base: that lane's first aggregate) into fp32 stages (S: d*dv floats, z: d
// floats).  Thread u of NT sums the S float4s u, u + NT, ... and, for
// u < d/4, z float4 u; the loads of four blocks are in flight together.
template <int NT>
__device__ __forceinline__ void sum_aggregates(const float4* base, int nsum, float* stage_s,
                                               float* stage_z, int u) {
  constexpr int E4 = E / 4, S4 = D * DV / 4, PER = (S4 + NT - 1) / NT;
  const bool has_z = u < D / 4;
  float4 acc[PER + 1];
#pragma unroll
  for (int e = 0; e <= PER; ++e) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
  for (int b0 = 0; b0 < nsum; b0 += 4) {
    float4 v[4][PER + 1];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (b0 + k < nsum) {
        const float4* blkp = base + (size_t)(b0 + k) * E4;
#pragma unroll
        for (int e = 0; e < PER; ++e)
          if (u + e * NT < S4) v[k][e] = __ldcg(blkp + u + e * NT);
        if (has_z) v[k][PER] = __ldcg(blkp + S4 + u);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (b0 + k < nsum) {
#pragma unroll
        for (int e = 0; e <= PER; ++e) {
          acc[e].x += v[k][e].x;
          acc[e].y += v[k][e].y;
          acc[e].z += v[k][e].z;
          acc[e].w += v[k][e].w;
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < PER; ++e)
    if (u + e * NT < S4) reinterpret_cast<float4*>(stage_s)[u + e * NT] = acc[e];
  if (has_z) reinterpret_cast<float4*>(stage_z)[u] = acc[PER];
}

// kCarry: the sequence is cut into several blocks and this launch starts
// each from the aggregates of the state launch.  Without it (one block per
// sequence, e.g. packed inputs) the carry code is left out of the image: the
// instruction working set of the warp roles matters to this kernel's speed.
// kTmaOut (dense non-causal launches): whole output tiles are staged in one
// of two staging tiles and written by TMA stores through a 4-D map (d, head,
// token, sequence) that clips a ragged last chunk at the sequence end; the
// other images have only the row stores.
template <bool kCarry, bool kTmaOut>
__global__ void __launch_bounds__(kThreads, 1)
    lt_block_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_o, const BlockArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  using Lo = BL<kTmaOut>;
  constexpr int NKV = Lo::NKV;
  __shared__ volatile int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int blk = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  int t0, ntok;
  if (!seq_bounds(a, s, t0, ntok)) {
    if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
    return;
  }
  const int nc = (ntok + kChunk - 1) / kChunk;
  const int c0 = blk * a.bc, c1 = min(c0 + a.bc, nc);
  if (c1 <= c0) return;  // nothing in this block (uniform over the CTA)
  const int Ri = c1 - c0;  // chunks of this block, walked in order
  const int G = a.G;
  const bool causal = a.causal != 0;
  const int n_items = Ri * G;
  // non-causal with a workspace: the state is the sum of all blocks and this
  // CTA reads only Q
  const bool nc_from_ws = !causal && a.ws != nullptr;

  uint8_t* sQ = smem + Lo::OFF_Q;
  uint8_t* sK = smem + Lo::OFF_KV;
  uint8_t* sV = smem + Lo::OFF_KV + KT;
  uint8_t* sSOP = smem + Lo::OFF_SOP;
  Bars bars = carve<NKV>(smem + Lo::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lo::OFF_BAR + Lo::NBARS * 8);

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
    mbar_init(bars.sop_full, 1);
    mbar_init(bars.sop_empty, 1);
    mbar_init(bars.s_full, 1);
    mbar_init(bars.s_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.p_full[i], 1);
      mbar_init(&bars.pb_full[i], 1);
      mbar_init(&bars.acc_full[i], 1);
      mbar_init(&bars.acc_empty[i], 1);
    }
    mbar_init(bars.drain, 1);
    fence_mbar_init();
  }
  init_ones_block(smem + Lo::OFF_ONES, tid, kThreads);
  fence_proxy_async_smem();
  if (warp == 17) tmem_alloc(tmem_slot, TM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_flag = &s_abort;
  // Carry: the aggregates of the earlier blocks (causal) or of every block
  // (non-causal), summed in fp32 in block order by warps 0-15 (the loads of
  // several blocks in flight at once) into the state operand buffer and the
  // z slot, which the state warps read after named barrier 4
  // (with a precomputed carry, slot blk alone)
  const int nprev =
      (!kCarry || a.ws == nullptr) ? 0 : (a.carry_pre ? 1 : (causal ? blk : a.nb));
  float* carry_s = reinterpret_cast<float*>(smem + Lo::OFF_SOP);
  float* carry_z = reinterpret_cast<float*>(smem + Lo::OFF_Z);
  if (kCarry && nprev > 0 && warp < 16) {
    sum_aggregates<512>(reinterpret_cast<const float4*>(a.ws) +
                            ((size_t)(s * a.Hkv + g) * a.nb + (a.carry_pre ? blk : 0)) * (E / 4),
                        nprev, carry_s, carry_z, tid);
    named_bar_sync(4, 512);
  }

  if (warp == 16) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      if (kTmaOut) prefetch_tmap(&tm_o);
      int q_issued = 0, kv_issued = 0;
      bool ok = true;
      auto load_kv = [&](int r) -> bool {
        const int st = r % NKV, c = c0 + r;
        if (!mbar_wait(&bars.kv_empty[st], ((r / NKV) & 1) ^ 1, abort_flag, a.err, kWaitLimitNs))
          return false;
        mbar_arrive_expect_tx(&bars.kv_full[st], KT + VT);
        tma_load_3d(sK + st * KVT, &tm_k, &bars.kv_full[st], 0, g, t0 + c * kChunk);
        tma_load_3d(sV + st * KVT, &tm_v, &bars.kv_full[st], 0, g, t0 + c * kChunk);
        ++kv_issued;
        return true;
      };
      auto load_q = [&](int j) -> bool {
        const int st = j % NQ, r = j / G, h = j % G, c = c0 + r;
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
        if (!nc_from_ws)
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
    __syncwarp();  // the whole warp reaches the final barrier together
  } else if (warp == 17) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_P = idesc_bf16_f32(kChunk, kChunk, 0, 0);
      constexpr uint32_t ID_SV = idesc_bf16_f32(D, DV + 16, 1, 1);
      constexpr uint32_t ID_PV = idesc_bf16_f32(kChunk, DV + 16, 0, 1);
      constexpr uint32_t ID_QS = idesc_bf16_f32(kChunk, DV + 16, 0, 1);
      // descriptor bases, advanced per stage / K step with one 64-bit add
      const uint64_t dQk = smem_desc_sw128(smem_u32(sQ), 16, 1024);      // K-major
      const uint64_t dKk = smem_desc_sw128(smem_u32(sK), 16, 1024);      // K-major
      const uint64_t dKmn = smem_desc_sw128(smem_u32(sK), kBox, 1024);   // MN-major
      const uint64_t dVmn = smem_desc_sw128(smem_u32(sV), kBox, 1024);   // MN-major V
      const uint32_t ones = smem_u32(smem + Lo::OFF_ONES);
      const uint64_t dSop = smem_desc_sw128(smem_u32(sSOP), D * kRowBytes, 1024);
      bool ok = true;
      // dS (or the running S for the non-causal state pass) = phi(K)^T [V | 1]
      auto issue_ds = [&](int r, uint32_t t_ds, bool accumulate) {
        const int st = r % NKV;
        // [V | 1]: the second 64-column group is the shared ones block
        const uint32_t va = smem_u32(sV) + st * KVT;
        const uint64_t ka = desc_advance(dKmn, st * KVT), vb = smem_desc_sw128(va, ones - va, 1024);
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
        // S_acc += dS of chunk r, once the state warpgroup has read S_<r
        // (phase r of s_empty; phase 0 is the carry it wrote).  Only chunks
        // before the block's last one feed a later state.
        auto state_mma = [&](int r) -> bool {
          if (r + 1 >= Ri) return true;
          if (!mbar_wait(&bars.kv_xf[r % NKV], (r / NKV) & 1, abort_flag, a.err, kWaitLimitNs) ||
              !mbar_wait(bars.s_empty, r & 1, abort_flag, a.err, kWaitLimitNs))
            return false;
          tc_fence_after();
          issue_ds(r, tmem + TM_S, true);
          umma_commit(bars.s_full);
          return true;
        };
        // score tile of item j into TMEM buffer j & 1.  The buffer last held
        // item j-2, whose P V MMAs were issued before this: the tensor pipe
        // runs them in order.
        auto score_mma = [&](int j) -> bool {
          const int r = j / G, qs = j % NQ;
          if (!mbar_wait(&bars.q_xf[qs], (j / NQ) & 1, abort_flag, a.err, kWaitLimitNs) ||
              !mbar_wait(&bars.kv_xf[r % NKV], (r / NKV) & 1, abort_flag, a.err, kWaitLimitNs))
            return false;
          tc_fence_after();
          const uint64_t qd = desc_advance(dQk, qs * QT);
          const uint64_t kd = desc_advance(dKk, (r % NKV) * KVT);
          const uint32_t t_p = tmem + TM_P + (j & 1) * kChunk;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk >> 2) * kBox + (kk & 3) * 32;
            umma_f16_ss(t_p, desc_advance(qd, o), desc_advance(kd, o), ID_P, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars.p_full[j & 1]);
          return true;
        };
        // item t's score tile (and the state product of its chunk) ahead of
        // item t-1's P V and phi(Q)[S|z]: the mask of item t then overlaps
        // those products.  Each step is issued from one place in the loop.
        for (int t = 0; t <= n_items && ok; ++t) {
          if (t < n_items) {
            ok = score_mma(t);
            if (ok && t % G == 0) ok = state_mma(t / G);
            if (!ok) break;
          }
          if (t == 0) continue;
          const int j = t - 1;
          const int r = j / G, h = j % G, qs = j % NQ, as = j & 1;
          const uint32_t va = smem_u32(sV) + (r % NKV) * KVT;
          const uint64_t vd = smem_desc_sw128(va, ones - va, 1024);  // [V | 1]
          const uint32_t t_acc = tmem + TM_ACC + as * ACCW;
          ok = mbar_wait(&bars.pb_full[as], (j >> 1) & 1, abort_flag, a.err, kWaitLimitNs) &&
               mbar_wait(&bars.acc_empty[as], ((j >> 1) & 1) ^ 1, abort_flag, a.err,
                         kWaitLimitNs);
          if (!ok) break;
          tc_fence_after();
          // P [V | 1]: bf16 scores from TMEM, 16 keys (8 columns) per MMA;
          // the ones column gives the row sums of the masked scores
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk)
            umma_f16_ts(t_acc, tmem + TM_P + as * kChunk + kk * 8, desc_advance(vd, kk * 2048),
                        ID_PV, kk > 0 ? 1u : 0u);
          if (h == G - 1) umma_commit(&bars.kv_empty[r % NKV]);
          if (h == 0) {
            ok = mbar_wait(bars.sop_full, r & 1, abort_flag, a.err, kWaitLimitNs);
            if (!ok) break;
            tc_fence_after();
          }
          issue_qs(t_acc, qs, true);
          umma_commit(&bars.acc_full[as]);
          umma_commit(&bars.q_empty[qs]);
          if (h == G - 1) umma_commit(bars.sop_empty);
        }
      } else {
        if (!nc_from_ws) {
          for (int r = 0; r < Ri && ok; ++r) {
            ok = mbar_wait(&bars.kv_xf[r % NKV], (r / NKV) & 1, abort_flag, a.err, kWaitLimitNs);
            if (!ok) break;
            tc_fence_after();
            issue_ds(r, tmem + TM_S, r > 0);
            umma_commit(&bars.kv_empty[r % NKV]);
          }
          if (ok) umma_commit(bars.s_full);
        }
        if (ok) ok = mbar_wait(bars.sop_full, 0, abort_flag, a.err, kWaitLimitNs);
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
    __syncwarp();
  } else if (warp < 8) {
    // ---------------------------------------------- transform warps
    const int x = tid;  // 0..255
    bool ok = true;
    // One loop over the tiles in arrival order (causal: K_r then the Q of
    // each head of chunk r; non-causal: every K, then every Q), so that the
    // transform code exists once in the kernel image.
    const int nkv = nc_from_ws ? 0 : Ri;
    const int T = causal ? Ri * (G + 1) : nkv + n_items;
    for (int t = 0; t < T && ok; ++t) {
      bool is_kv;
      int r, j;
      if (causal) {
        r = t / (G + 1);
        const int k = t - r * (G + 1);
        is_kv = k == 0;
        j = r * G + k - 1;
      } else {
        is_kv = t < nkv;
        r = t;
        j = t - nkv;
      }
      const int st = is_kv ? r % NKV : j % NQ;
      const uint32_t par = is_kv ? (r / NKV) & 1 : (j / NQ) & 1;
      ok = mbar_wait(is_kv ? &bars.kv_full[st] : &bars.q_full[st], par, abort_flag, a.err,
                     kWaitLimitNs);
      if (!ok) break;
      uint8_t* tile = is_kv ? sK + st * KVT : sQ + st * QT;
      // Q rows past the end of the sequence only feed output rows that are
      // never stored, so a Q tile is always transformed whole
      const int valid = is_kv ? min(kChunk, ntok - (c0 + r) * kChunk) : kChunk;
      if (valid >= kChunk) {
        phi_tile_full<D / 64, kXf>(tile, x);
      } else {
        // ragged end: phi on K with the rows past it zeroed, and those V rows zeroed
#pragma unroll 1
        for (int u = 0; u < 2; ++u) xf_tile<D / 64, kXf>(tile + u * KT, valid, u == 0, x);
      }
      fence_proxy_async_smem();
      named_bar_sync(1, kXf);
      if (x == 0) mbar_arrive(is_kv ? &bars.kv_xf[st] : &bars.q_xf[st]);
    }
  } else if (warp < 12) {
    // ---------------------------------------------------- mask warpgroup
    const int x = tid - 256, sp = warp & 3;
    const int row = sp * 32 + lane;  // TMEM lane == chunk row
    const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
    bool ok = true;
    // causal mask and bf16 rounding of the score tile, in place in TMEM:
    // fp32 columns [32b, 32b+32) become packed bf16 columns [16b, 16b+16),
    // which only overwrites columns this thread has already read
    auto mask_p = [&](int j) -> bool {
      const int as = j & 1;
      if (!mbar_wait(&bars.p_full[as], (j >> 1) & 1, abort_flag, a.err, kWaitLimitNs))
        return false;
      tc_fence_after();
      const uint32_t lane_sel = (uint32_t)(sp * 32) << 16;
      const uint32_t t_p = tmem + TM_P + as * kChunk + lane_sel;
#pragma unroll
      for (int b = 0; b < kChunk / 32; ++b) {
        uint32_t pk[16];
        if (b <= sp) {  // warp-uniform: blocks right of the diagonal are all zero
          float r[32];
          tmem_ld32(t_p + b * 32, r);
          tmem_wait_ld();
          if (b < sp) {  // block entirely left of the diagonal
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(r[2 * e], r[2 * e + 1]);
          } else {  // the diagonal block
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float lo = (b * 32 + 2 * e > row) ? 0.0f : r[2 * e];
              const float hi = (b * 32 + 2 * e + 1 > row) ? 0.0f : r[2 * e + 1];
              pk[e] = pack_bf16x2(lo, hi);
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        }
        tmem_st16(t_p + b * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      named_bar_sync(2, 128);
      if (x == 0) mbar_arrive(&bars.pb_full[as]);
      return true;
    };
    auto epilogue = [&](int j) -> bool {
      const int r = j / G, h = j % G, as = j & 1, c = c0 + r;
      if (!mbar_wait(&bars.acc_full[as], (j >> 1) & 1, abort_flag, a.err, kWaitLimitNs))
        return false;
      tc_fence_after();
      const uint32_t t_acc = tmem + TM_ACC + as * ACCW + lane_base;
      // numerator columns -> normalised packed bf16, 32 at a time; the
      // accumulator is released before the stores
      uint32_t pk[DV / 2];
      float inv;
      {
        float n[32];
        const float den = tmem_ld1(t_acc + DV);
        tmem_ld32(t_acc, n);
        tmem_wait_ld();
        inv = 1.0f / (den + a.eps);
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(n[2 * e] * inv, n[2 * e + 1] * inv);
      }
#pragma unroll
      for (int cb = 1; cb < DV / 32; ++cb) {
        float n[32];
        tmem_ld32(t_acc + cb * 32, n);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[cb * 16 + e] = pack_bf16x2(n[2 * e] * inv, n[2 * e + 1] * inv);
      }
      if (kTmaOut) {
        // staging tile j & 1 was last stored from by item j-2: its reads are
        // done once at most one bulk group (item j-1's) is pending
        if (x == 0 && j >= 2) bulk_wait_read_but_last();
      }
      tc_fence_before();
      named_bar_sync(2, 128);
      if (x == 0) mbar_arrive(&bars.acc_empty[as]);
      if (kTmaOut) {
        uint8_t* tile = smem + Lo::OFF_OST + (j & 1) * OSTT;
#pragma unroll
        for (int q = 0; q < DV / 8; ++q)
          *reinterpret_cast<uint4*>(tile + sw128_off(row, q)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        fence_proxy_async_smem();
        named_bar_sync(2, 128);
        if (x == 0) {
          tma_store_4d(&tm_o, tile, 0, g * G + h, c * kChunk, s);
          bulk_commit_group();
        }
      } else {
        const int valid = min(kChunk, ntok - c * kChunk);
        if (row < valid) {
          uint4* orow = reinterpret_cast<uint4*>(
              a.out + ((size_t)(t0 + c * kChunk + row) * a.Hq + (size_t)(g * G + h)) * DV);
#pragma unroll
          for (int q = 0; q < DV / 8; ++q)
            orow[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      return true;
    };
    // the mask of item j+1 goes before the epilogue of item j: the mask is on
    // the path to the next MMAs, the epilogue only drains
    for (int t = 0; t <= n_items && ok; ++t) {
      if (causal && t < n_items) ok = mask_p(t);
      if (ok && t > 0) ok = epilogue(t - 1);
    }
    if (kTmaOut && x == 0) bulk_wait_all();  // every output store has landed
  } else if (warp < 16) {
    // -------------------------------------------------- state warpgroup
    // The running [S | z] is an fp32 M=64 accumulator in TMEM (S_acc): state
    // row a = 16*sp + l lives in lane l < 16 of sub-partition sp.  This
    // group writes the carry into it, and before every chunk copies it,
    // rounded to bf16, into the MN-major [S | z 0 ..] operand.
    const int y = tid - 384, sp = warp & 3;
    const uint32_t t_s = tmem + TM_S + ((uint32_t)(sp * 32) << 16);
    const bool has_row = lane < 16;
    const int row = sp * 16 + lane;
    bool ok = true;
    uint32_t w[ACCW / 2];  // this thread's row of [S | z 0 ..], packed bf16
    // carry: the staged sum (zero without earlier blocks) into S_acc
    auto load_carry = [&]() {
#pragma unroll 1
      for (int q = 0; q < ACCW / 16; ++q) {
        float c[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) c[e] = 0.0f;
        if (kCarry && nprev > 0 && has_row) {
          if (q < DV / 16) {
            const float4* r4 = reinterpret_cast<const float4*>(carry_s + row * DV + q * 16);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float4 v = r4[u];
              c[4 * u] = v.x;
              c[4 * u + 1] = v.y;
              c[4 * u + 2] = v.z;
              c[4 * u + 3] = v.w;
            }
          } else {
            c[0] = carry_z[row];
          }
        }
        uint32_t u16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) u16[e] = __float_as_uint(c[e]);
        tmem_st16(t_s + q * 16, u16);
      }
      tmem_wait_st();
    };
    // S_acc -> w, rounded to bf16
    auto read_state = [&]() {
#pragma unroll
      for (int q = 0; q < ACCW / 16; ++q) {
        float c[16];
        tmem_ld16(t_s + q * 16, c);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) w[q * 8 + e] = pack_bf16x2(c[2 * e], c[2 * e + 1]);
      }
    };
    // Causal: step r publishes [S|z]_<r for chunk r; step 0 starts S_acc from
    // the carry, step r > 0 reads it once the state product of chunk r-1 has
    // landed, then releases it (phase r of s_empty) for the product of chunk
    // r.  Non-causal: one step, with the carry or the state of this block.
    const int nsteps = causal ? Ri : 1;
    for (int r = 0; r < nsteps && ok; ++r) {
      if (r == 0 && (causal || nc_from_ws)) {
        load_carry();
      } else {
        ok = mbar_wait(bars.s_full, (causal ? r - 1 : 0) & 1, abort_flag, a.err, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after();
      }
      read_state();
      tc_fence_before();
      // also orders every thread's read of the staged carry (in the operand
      // buffer) before the operand is written
      named_bar_sync(3, 128);
      if (causal && y == 0) mbar_arrive(bars.s_empty);
      // w -> the operand (pieces of 8 columns; columns dv.. are [z 0 ..])
      ok = mbar_wait(bars.sop_empty, (r & 1) ^ 1, abort_flag, a.err, kWaitLimitNs);
      if (!ok) break;
      if (has_row) {
#pragma unroll
        for (int q8 = 0; q8 < ACCW / 8; ++q8)
          *reinterpret_cast<uint4*>(sSOP + (q8 >> 3) * (D * kRowBytes) + sw128_off(row, q8 & 7)) =
              make_uint4(w[4 * q8], w[4 * q8 + 1], w[4 * q8 + 2], w[4 * q8 + 3]);
      }
      fence_proxy_async_smem();
      named_bar_sync(3, 128);
      if (y == 0) mbar_arrive(bars.sop_full);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 17) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace

bool block_supported(const FwdLaunch& p) { return p.d == 64 && p.dv == 64; }

namespace {
cudaError_t launch_block(const FwdLaunch& p, int nb, const float* ws, bool carry_pre,
                         cudaStream_t stream) {
  CUtensorMap tq, tk, tv, to;
  // TMA stores for dense non-causal launches: in causal mode the epilogue
  // shares warps with the mask, which is on the chunk chain, and the fourth
  // K/V stage matters to packed inputs
  const bool tma_out = p.cu_seqlens == nullptr && p.causal == 0;
  if (!make_tmap_3d(&tq, p.q, D, p.Hq, p.total_tokens, 64) ||
      !make_tmap_3d(&tk, p.k, D, p.Hkv, p.total_tokens, 64) ||
      !make_tmap_3d(&tv, p.v, DV, p.Hkv, p.total_tokens, 64) ||
      (tma_out ? !make_tmap_4d_dense(&to, p.out, DV, p.Hq, p.N, p.B, 64)
               : !make_tmap_3d(&to, p.out, DV, p.Hq, p.total_tokens, 64)))
    return cudaErrorInvalidValue;
  BlockArgs a;
  a.out = reinterpret_cast<__nv_bfloat16*>(p.out);
  a.cu_seqlens = p.cu_seqlens;
  a.ws = (nb > 1 || carry_pre) ? const_cast<float*>(ws) : nullptr;
  a.carry_pre = carry_pre ? 1 : 0;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.N = p.N;
  a.G = p.Hq / p.Hkv;
  a.causal = p.causal;
  a.nb = nb;
  a.bc = block_chunks(p, nb);
  a.eps = p.eps;
  a.total_tokens = (int)p.total_tokens;
  a.err = p.err;
  auto fk = a.ws != nullptr
                ? (tma_out ? lt_block_fwd_kernel<true, true> : lt_block_fwd_kernel<true, false>)
                : (tma_out ? lt_block_fwd_kernel<false, true> : lt_block_fwd_kernel<false, false>);
  const int smem = tma_out ? BL<true>::SMEM : BL<false>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(fk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  fk<<<dim3(nb, p.Hkv, p.B), kThreads, smem, stream>>>(tq, tk, tv, to, a);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_fwd_bf16_block(const FwdLaunch& p, int nb, const float* ws,
                                  cudaStream_t stream) {
  return launch_block(p, nb, ws, false, stream);
}

cudaError_t launch_fwd_bf16_block_pre(const FwdLaunch& p, int nb, const float* ws,
                                      cudaStream_t stream) {
  return launch_block(p, nb, ws, true, stream);
}

}  // namespace lt
