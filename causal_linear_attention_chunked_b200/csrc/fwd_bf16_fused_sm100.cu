// fwd_bf16_fused_sm100.cu -- one-launch chunked linear attention for short
// blocks, bf16 I/O with fp32 accumulation, d = dv = 64 (sm_100a: tcgen05 +
// TMA + TMEM).
//
// Method (lineartile 1.0.0, "How It Works" and "Reference"):
//     O_i = phi(Q_i) S_i / (phi(Q_i) . z_i + eps),  S_i = sum_{j<=i} phi(K_j)^T V_j,
//     z_i = sum_{j<=i} phi(K_j),  phi(x) = ELU(x) + 1.
// Evaluation is the two-level chunked scan of "Why Stream Wins at
// Ultra-Long Context", section 5.3 (chunk-local work, an inter-chunk carry,
// and a broadcast correction), in ONE cooperative launch: a sequence is cut
// into nb blocks of at most four 128-token chunks, one CTA per block (all
// resident at once), and each CTA
//   1. loads every K/V tile of its block once (they stay in the ring),
//      applies phi to K and reduces its block aggregate
//          A_b = sum_{c in b} phi(K_c)^T [V_c | 1]         (fp32, TMEM)
//      on the tensor cores (phase A), and publishes it to the workspace;
//   2. meets every other CTA at a grid barrier, then sums the aggregates of
//      the blocks before it (causal) or of all blocks (non-causal) in block
//      order -- the same products and summation order as the two-launch
//      path, so the two agree bit for bit;
//   3. walks its chunks from that carry, carrying [S|z] += phi(K_c)^T [V_c|1]
//      in TMEM, and computes
//         num_c = mask(phi(Q_c) phi(K_c)^T) V_c + phi(Q_c) S_<c
//         den_c = mask(phi(Q_c) phi(K_c)^T) 1   + phi(Q_c) z_<c
//      with the normaliser as the extra column of P [V | 1] and phi(Q) [S | z].
// The score, mask and intra-chunk products of the first chunks proceed while
// the aggregates are exchanged.
//
// Warp roles (608 threads; TMEM sub-partition = warp % 4):
//   warps 0-7   transform: phi in place on K and Q tiles (tail rows zeroed);
//               with the state warps, the carry sum
//   warps 8-11  mask + epilogue: causal mask of the score tile, bf16 in
//               place in TMEM; accumulator -> normalised bf16 rows -> global
//   warps 12-15 state: publish the aggregate, gather the carry into the TMEM
//               state accumulator, and before every chunk copy the state,
//               rounded to bf16, into a [S | z] B operand (two buffers)
//   warp 16     TMA producer
//   warp 17     TMEM allocator; issues the score, P V and phi(Q)[S|z] products
//   warp 18     issues phase A and the state products
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

constexpr int D = 64, DV = 64;
constexpr int E = D * DV + D;  // block aggregate: S (row-major d x dv) then z
constexpr int QT = kChunk * D * 2, KT = kChunk * D * 2, VT = kChunk * DV * 2;
constexpr int KVT = KT + VT;  // one K/V stage: [K][V]
constexpr int SOPT = (DV / 64 + 1) * D * kRowBytes;
constexpr int ONEST = kChunk * kRowBytes;
constexpr int ACCW = DV + 16;

struct FusedArgs {
  __nv_bfloat16* out;
  const int32_t* cu_seqlens;
  float* ws;        // block aggregates [lane][nb][E], or nullptr
  int Hq, Hkv, N, G, causal;
  int nb;           // blocks per sequence (lane)
  int bc;           // chunks per block
  float eps;
  int total_tokens;
  int* err;
};

__device__ __forceinline__ bool seq_bounds(const FusedArgs& a, int s, int& t0, int& n) {
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
constexpr int kThreads = 608;
constexpr int kXf = 256;  // transform threads (warps 0-7, two per SM sub-partition)
constexpr int NKV = 4;
// two score tiles (item j uses j & 1), two accumulators, the running state
constexpr int TM_P = 0, TM_ACC = 2 * kChunk, TM_S = TM_ACC + 2 * ACCW, TM_COLS = 512;
static_assert(TM_S + ACCW <= TM_COLS, "TMEM budget");
// Shared-memory layout for NQ Q stages and NSOP state operand buffers (the
// one-launch mode trades a Q stage for a second operand buffer).  The carry
// sum is staged in operand buffer 0 (S) and the z slot.
template <int NQ, int NSOP>
struct Layout {
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + NQ * QT;  // stage st: [K][V] at st*KVT
  static constexpr int OFF_ONES = OFF_KV + NKV * KVT;
  static constexpr int OFF_SOP = OFF_ONES + ONEST;
  static constexpr int OFF_Z = OFF_SOP + NSOP * SOPT;
  static constexpr int OFF_BAR = OFF_Z + D * 4;
  static constexpr int NBARS = 3 * NQ + 3 * NKV + 2 * 2 + 2 * NSOP + 2 + 2 * 2 + 1 + 2;
  static constexpr int SMEM = OFF_BAR + NBARS * 8 + 16 + 1024;
  static_assert(SOPT >= D * DV * 4, "the carry's S is staged in an operand buffer");
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct Bars {
  uint64_t *q_full, *q_empty, *q_xf, *kv_full, *kv_empty, *kv_xf;
  uint64_t *p_full, *pb_full, *sop_full, *sop_empty;
  uint64_t *s_full, *s_empty, *acc_full, *acc_empty, *drain;
  uint64_t* agg_full;  // phase A: the block aggregate is in S_acc
  uint64_t* drain2;    // the state issuer's products are complete
};

template <int NQ, int NSOP>
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
  r.sop_full = b; b += NSOP;
  r.sop_empty = b; b += NSOP;
  r.s_full = b++;
  r.s_empty = b++;
  r.acc_full = b; b += 2;
  r.acc_empty = b; b += 2;
  r.drain = b++;
  r.agg_full = b++;
  r.drain2 = b++;
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
  // S is staged with the float4 index of a row XOR-ed with the row, so that
  // the state warps, one row per thread, read it without bank conflicts
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int i = u + e * NT;
    if (i < S4) reinterpret_cast<float4*>(stage_s)[(i & ~15) | ((i ^ (i >> 4)) & 15)] = acc[e];
  }
  if (has_z) reinterpret_cast<float4*>(stage_z)[u] = acc[PER];
}

// NQ Q stages and NSOP state operand buffers (shared-memory layout).  The
// main issuer (warp 17) polls, so that a product whose inputs are ready never
// waits behind one whose inputs are late; the state products have their own
// issuer (warp 18).
template <int NQ, int NSOP>
__global__ void __launch_bounds__(kThreads, 1)
    lt_fused_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const FusedArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  using L = Layout<NQ, NSOP>;
  __shared__ volatile int s_abort;
  __shared__ volatile int s_me_next;  // mask/epilogue warps: the step thread 0 chose
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int blk = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  int t0, ntok;
  if (!seq_bounds(a, s, t0, ntok)) {
    if (tid == 0) report_error(a.err, kDevErrBadSeqlens);
    return;
  }
  const int nc = (ntok + kChunk - 1) / kChunk;
  const int c0 = blk * a.bc, c1 = min(c0 + a.bc, nc);
  if (c1 <= c0) return;  // never: the host plans no empty block (every CTA must arrive at the grid barrier)
  const int Ri = c1 - c0;  // chunks of this block, walked in order
  const int G = a.G;
  const bool causal = a.causal != 0;
  const int n_items = Ri * G;
  // non-causal with a workspace: the state is the sum of all blocks and this
  // CTA reads only Q
  // this CTA first reduces its block's K, V to the aggregate (phase A) and
  // publishes it, then gathers the carry from the aggregates the other CTAs
  // publish; the K/V ring holds every chunk of the block, so each tile is
  // loaded once.  Non-causal: the whole state is the carry.

  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_KV;
  uint8_t* sV = smem + L::OFF_KV + KT;
  uint8_t* sSOP = smem + L::OFF_SOP;
  Bars bars = carve<NQ, NSOP>(smem + L::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + L::NBARS * 8);

  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&bars.q_full[i], 1);
      mbar_init(&bars.q_empty[i], 1);
      mbar_init(&bars.q_xf[i], 1);
    }
    for (int i = 0; i < NKV; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      // causal: released by the main issuer (scores, P V) and the state issuer
      mbar_init(&bars.kv_empty[i], causal ? 2 : 1);
      mbar_init(&bars.kv_xf[i], 1);
    }
    for (int i = 0; i < NSOP; ++i) {
      mbar_init(&bars.sop_full[i], 1);
      mbar_init(&bars.sop_empty[i], 1);
    }
    mbar_init(bars.s_full, 1);
    mbar_init(bars.s_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.p_full[i], 1);
      mbar_init(&bars.pb_full[i], 1);
      mbar_init(&bars.acc_full[i], 1);
      mbar_init(&bars.acc_empty[i], 1);
    }
    mbar_init(bars.drain, 1);
    mbar_init(bars.agg_full, 1);
    mbar_init(bars.drain2, 1);
    fence_mbar_init();
  }
  init_ones_block(smem + L::OFF_ONES, tid, kThreads);
  fence_proxy_async_smem();
  if (warp == 17) tmem_alloc(tmem_slot, TM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_flag = &s_abort;

  // Carry: the aggregates of the earlier blocks (causal) or of every block
  // (non-causal), summed in fp32 in block order into the state operand
  // buffers (free until the state warps first stage [S|z]).  Warps 0-15
  // share the work so that the loads of several blocks are in flight at
  // once; the state warps read the sum after named barrier 4.
  // the number of aggregates in the carry, and where this lane's aggregates
  // start; the sum is staged (fp32) in the state operand buffers, free until
  // the state warps first stage [S|z]
  const int nprev = a.ws == nullptr ? 0 : (causal ? blk : a.nb);
  const float4* agg_base =
      a.ws == nullptr ? nullptr
                      : reinterpret_cast<const float4*>(a.ws) + (size_t)(s * a.Hkv + g) * a.nb * (E / 4);
  float* carry_stage = reinterpret_cast<float*>(smem + L::OFF_SOP);
  float* carry_stage_z = reinterpret_cast<float*>(smem + L::OFF_Z);
  // The transform warps and the state warps (384 threads) sum the aggregates
  // between two barriers 5, once the state warps have passed the grid
  // barrier.  Both groups pass both barriers on every path (an abort skips
  // only the loads), so no barrier is left waiting.
  const bool gather = nprev > 0;
  auto gather_part = [&](int u) {
    named_bar_sync(5, 384);
    if (!*abort_flag) sum_aggregates<384>(agg_base, nprev, carry_stage, carry_stage_z, u);
    named_bar_sync(5, 384);
  };

  if (warp == 16) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
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
      // every K/V tile first (phase A needs them), then the Q tiles
      for (int r = 0; r < Ri && ok; ++r) ok = load_kv(r);
      for (int j = 0; j < n_items && ok; ++j) ok = load_q(j);
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
      const uint32_t ones = smem_u32(smem + L::OFF_ONES);
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
      auto issue_qs = [&](uint32_t t_acc, int qs, int sb, bool accumulate) {
        const uint64_t qa = desc_advance(dQk, qs * QT);
        const uint64_t sd = desc_advance(dSop, sb * SOPT);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_f16_ss(t_acc, desc_advance(qa, (kk >> 2) * kBox + (kk & 3) * 32),
                      desc_advance(sd, kk * 2048), ID_QS, (accumulate || kk > 0) ? 1u : 0u);
      };
      if (causal) {
        // Per item j (chunk r = j / G, head h = j % G), in program order:
        //   SC(j)  score tile into TMEM buffer j & 1 (the buffer last held
        //          item j-2, whose P V was issued before: the pipe is in order)
        //   PV(j)  Acc(j & 1) = P [V | 1] once the mask warps have rounded P
        //          and the epilogue has drained the accumulator
        //   QS(j)  Acc(j & 1) += phi(Q) [S | z]_<r once the operand is staged
        // Split: the state products run on their own issuer (warp 18) and
        // the K/V stage is released by both issuers; otherwise this thread
        // issues them too.
        auto score_ready = [&](int t) {
          const int r = t / G;
          return mbar_test(&bars.q_xf[t % NQ], (t / NQ) & 1) &&
                 mbar_test(&bars.kv_xf[r % NKV], (r / NKV) & 1);
        };
        auto score = [&](int t) {
          const int r = t / G, q = t % NQ;
          const uint64_t qd = desc_advance(dQk, q * QT);
          const uint64_t kd = desc_advance(dKk, (r % NKV) * KVT);
          const uint32_t t_p = tmem + TM_P + (t & 1) * kChunk;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk >> 2) * kBox + (kk & 3) * 32;
            umma_f16_ss(t_p, desc_advance(qd, o), desc_advance(kd, o), ID_P, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars.p_full[t & 1]);
        };
        // Issue by polling, so that products whose inputs are ready never
        // wait behind one whose inputs are late (the first items' scores,
        // masks and P V run while the carry is still being gathered):
        //   QS(j)  once P V(j) is issued and the chunk's operand is staged
        //   SC(j)  once its tiles are ready and P V(j-2) (the last user of
        //          TMEM buffer j & 1) is issued
        //   PV(j)  once the mask warps have rounded P(j) and the epilogue has
        //          drained accumulator j & 1
        int sc = 0, pv = 0, qn = 0;
        uint32_t idle = 0;
        uint64_t idle_t0 = 0;
        while (qn < n_items && ok) {
          bool did = false;
          if (qn < pv && (qn % G != 0 || mbar_test(&bars.sop_full[(qn / G) % NSOP],
                                                     ((qn / G) / NSOP) & 1))) {
            tc_fence_after();
            const int r = qn / G, h = qn % G, as = qn & 1;
            issue_qs(tmem + TM_ACC + as * ACCW, qn % NQ, r % NSOP, true);
            umma_commit(&bars.acc_full[as]);
            umma_commit(&bars.q_empty[qn % NQ]);
            if (h == G - 1) umma_commit(&bars.sop_empty[r % NSOP]);
            ++qn;
            did = true;
          } else if (sc < n_items && sc <= pv + 1 && score_ready(sc)) {
            tc_fence_after();
            score(sc);
            ++sc;
            did = true;
          } else if (pv < sc && mbar_test(&bars.pb_full[pv & 1], (pv >> 1) & 1) &&
                     mbar_test(&bars.acc_empty[pv & 1], ((pv >> 1) & 1) ^ 1)) {
            tc_fence_after();
            const int r = pv / G, h = pv % G, as = pv & 1;
            const uint32_t va = smem_u32(sV) + (r % NKV) * KVT;
            const uint64_t vd = smem_desc_sw128(va, ones - va, 1024);  // [V | 1]
            const uint32_t t_acc = tmem + TM_ACC + as * ACCW;
            // P [V | 1]: bf16 scores from TMEM, 16 keys (8 columns) per MMA;
            // the ones column gives the row sums of the masked scores
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk)
              umma_f16_ts(t_acc, tmem + TM_P + as * kChunk + kk * 8, desc_advance(vd, kk * 2048),
                          ID_PV, kk > 0 ? 1u : 0u);
            if (h == G - 1) umma_commit(&bars.kv_empty[r % NKV]);
            ++pv;
            did = true;
          }
          if (did) {
            idle = 0;
          } else if ((++idle & 255u) == 0) {
            if (*abort_flag) {
              ok = false;
            } else if (idle == 256) {
              idle_t0 = global_timer_ns();
            } else if (global_timer_ns() - idle_t0 > kWaitLimitNs) {
              *abort_flag = 1;
              report_error(a.err, kDevErrTimeout);
              ok = false;
            }
          }
        }
      } else {
        // non-causal: the whole state is the carry, staged once
        if (ok) ok = mbar_wait(&bars.sop_full[0], 0, abort_flag, a.err, kWaitLimitNs);
        for (int j = 0; j < n_items && ok; ++j) {
          const int qs = j % NQ, as = j & 1;
          ok = mbar_wait(&bars.q_xf[qs], (j / NQ) & 1, abort_flag, a.err, kWaitLimitNs) &&
               mbar_wait(&bars.acc_empty[as], ((j >> 1) & 1) ^ 1, abort_flag, a.err,
                         kWaitLimitNs);
          if (!ok) break;
          tc_fence_after();
          issue_qs(tmem + TM_ACC + as * ACCW, qs, 0, false);
          umma_commit(&bars.acc_full[as]);
          umma_commit(&bars.q_empty[qs]);
        }
      }
      umma_commit(bars.drain);
      int dummy = 0;
      mbar_wait(bars.drain, 0, &dummy, nullptr, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp == 18) {
    // ------------------------------------------------ state-product issuer
    // Fused mode: phase A, S_acc = sum_r phi(K_r)^T [V_r | 1] (the block
    // aggregate).  Causal: S_acc += phi(K_r)^T [V_r | 1] for each chunk but
    // the last, once the state warps have read S_<r (phase r of s_empty),
    // then this issuer's share of the K/V stage release.
    if (lane == 0) {
      constexpr uint32_t ID_SV = idesc_bf16_f32(D, DV + 16, 1, 1);
      const uint64_t dKmn = smem_desc_sw128(smem_u32(sK), kBox, 1024);  // MN-major phi(K)
      const uint32_t ones = smem_u32(smem + L::OFF_ONES);
      auto issue_ds = [&](int r, bool accumulate) {
        const int st = r % NKV;
        // [V | 1]: the second 64-column group is the shared ones block
        const uint32_t va = smem_u32(sV) + st * KVT;
        const uint64_t ka = desc_advance(dKmn, st * KVT), vb = smem_desc_sw128(va, ones - va, 1024);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          umma_f16_ss(tmem + TM_S, desc_advance(ka, kk * 2048), desc_advance(vb, kk * 2048), ID_SV,
                      (accumulate || kk > 0) ? 1u : 0u);
      };
      bool ok = true;
      for (int r = 0; r < Ri && ok; ++r) {
        ok = mbar_wait(&bars.kv_xf[r % NKV], (r / NKV) & 1, abort_flag, a.err, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after();
        issue_ds(r, r > 0);
      }
      if (ok) umma_commit(bars.agg_full);
      if (causal) {
        for (int r = 0; r < Ri && ok; ++r) {
          if (r + 1 < Ri) {
            ok = mbar_wait(bars.s_empty, r & 1, abort_flag, a.err, kWaitLimitNs) &&
                 mbar_wait(&bars.kv_xf[r % NKV], (r / NKV) & 1, abort_flag, a.err, kWaitLimitNs);
            if (!ok) break;
            tc_fence_after();
            issue_ds(r, true);
            umma_commit(bars.s_full);
            umma_commit(&bars.kv_empty[r % NKV]);
          } else {
            mbar_arrive(&bars.kv_empty[r % NKV]);  // the last chunk feeds no state
          }
        }
      }
      umma_commit(bars.drain2);
      int dummy = 0;
      mbar_wait(bars.drain2, 0, &dummy, nullptr, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ---------------------------------------------- transform warps
    const int x = tid;  // 0..255
    bool ok = true;
    // One loop over the tiles in arrival order (every K, then every Q), so
    // that the transform code exists once in the kernel image.  The gather
    // comes before the last Q tile that is loaded without waiting on a
    // product: by then the grid barrier has usually passed, and that tile's
    // item waits for an accumulator that needs the carry anyway.
    const int nkv = Ri;
    const int T = nkv + n_items;
    const int join_t = nkv + max(0, min(n_items, NQ) - 2);
    bool joined = !gather;
    for (int t = 0; t < T && ok; ++t) {
      const bool is_kv = t < nkv;
      const int r = t, j = t - nkv;
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
      if (!joined && t == join_t) {
        gather_part(x);
        joined = true;
      }
    }
    if (!joined) gather_part(x);  // after an abort: keep the barrier sequence
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
      tc_fence_before();
      named_bar_sync(2, 128);
      if (x == 0) mbar_arrive(&bars.acc_empty[as]);
      const int valid = min(kChunk, ntok - c * kChunk);
      if (row < valid) {
        uint4* orow = reinterpret_cast<uint4*>(
            a.out + ((size_t)(t0 + c * kChunk + row) * a.Hq + (size_t)(g * G + h)) * DV);
#pragma unroll
        for (int q = 0; q < DV / 8; ++q)
          orow[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
      return true;
    };
    // Masks and epilogues in whichever order their inputs arrive (a mask
    // whose score tile is ready never waits behind an epilogue whose
    // accumulator needs the carry).  Thread 0 polls and picks the step; the
    // group barrier at the end of every step orders the next pick after
    // everyone has read this one.  Masks go first when both are ready.
    int mt = 0, et = 0;
    while (et < n_items && ok) {
      if (x == 0) {
        int c = -1;
        uint32_t spins = 0;
        uint64_t w0 = 0;
        while (c < 0) {
          if (causal && mt < n_items && mbar_test(&bars.p_full[mt & 1], (mt >> 1) & 1)) {
            c = 0;
          } else if (et < (causal ? mt : n_items) &&
                     mbar_test(&bars.acc_full[et & 1], (et >> 1) & 1)) {
            c = 1;
          } else if ((++spins & 255u) == 0) {
            if (*abort_flag) {
              c = 2;
            } else if (spins == 256) {
              w0 = global_timer_ns();
            } else if (global_timer_ns() - w0 > kWaitLimitNs) {
              *abort_flag = 1;
              report_error(a.err, kDevErrTimeout);
              c = 2;
            }
          }
        }
        s_me_next = c;
      }
      named_bar_sync(2, 128);
      const int c = s_me_next;
      if (c == 2) {
        ok = false;
      } else if (c == 0) {
        ok = mask_p(mt++);
      } else {
        ok = epilogue(et++);
      }
    }
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
    const float* cS = carry_stage;
    const float* cZ = carry_stage_z;
    const bool have_carry = nprev > 0;
    // Fused mode, before the first chunk: S_acc holds this block's aggregate
    // (phase A).  Publish it to the workspace (causal: unless this is the
    // last block, whose aggregate no block needs); every CTA arrives once at
    // the grid barrier, on every path; a CTA with a carry waits there, then
    // sums the aggregates together with the transform warps.
    auto publish_and_gather = [&](bool do_gather) {
      const bool pok = mbar_wait(bars.agg_full, 0, abort_flag, a.err, kWaitLimitNs);
      tc_fence_after();
      if (pok && (!causal || blk + 1 < a.nb)) {
        float* dst = a.ws + ((size_t)(s * a.Hkv + g) * a.nb + blk) * E;
#pragma unroll
        for (int q = 0; q < ACCW / 16; ++q) {
          float c[16];
          tmem_ld16(t_s + q * 16, c);
          tmem_wait_ld();
          if (has_row) {
            if (q < DV / 16) {
              float4* d4 = reinterpret_cast<float4*>(dst + row * DV + q * 16);
#pragma unroll
              for (int u = 0; u < 4; ++u)
                d4[u] = make_float4(c[4 * u], c[4 * u + 1], c[4 * u + 2], c[4 * u + 3]);
            } else {
              dst[D * DV + row] = c[0];
            }
          }
        }
      }
      tc_fence_before();
      // the group barrier orders every thread's aggregate writes before the
      // arriving thread's release at gpu scope (release is cumulative)
      named_bar_sync(3, 128);
      if (y == 0) grid_barrier(do_gather, abort_flag, a.err, kWaitLimitNs);
      if (do_gather) gather_part(256 + y);
    };
    // step 0: the carry (zero without earlier blocks) -> w and, in causal
    // mode, the starting value of S_acc
    auto load_carry = [&]() {
#pragma unroll
      for (int q = 0; q < ACCW / 16; ++q) {
        float c[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) c[e] = 0.0f;
        if (have_carry && has_row) {
          if (q < DV / 16) {
            const float4* r4 = reinterpret_cast<const float4*>(cS) + row * (DV / 4);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float4 v = r4[(q * 4 + u) ^ (row & 15)];
              c[4 * u] = v.x;
              c[4 * u + 1] = v.y;
              c[4 * u + 2] = v.z;
              c[4 * u + 3] = v.w;
            }
          } else {
            c[0] = cZ[row];
          }
        }
        if (causal) {
          uint32_t u16[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) u16[e] = __float_as_uint(c[e]);
          tmem_st16(t_s + q * 16, u16);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) w[q * 8 + e] = pack_bf16x2(c[2 * e], c[2 * e + 1]);
      }
      if (causal) tmem_wait_st();
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
    // The operand of chunk r goes to buffer r % NSOP, so staging chunk r
    // waits only for the last product that read chunk r - NSOP's operand.
    // Step 0 reads the carry from the operand buffers themselves: barrier 3
    // below orders every thread's read before the first operand write.
    // causal block 0 has no carry but publishes its aggregate
    publish_and_gather(gather);
    ok = !*abort_flag;
    const int nsteps = causal ? Ri : 1;
    for (int r = 0; r < nsteps && ok; ++r) {
      if (r == 0) {
        load_carry();
      } else {
        ok = mbar_wait(bars.s_full, (causal ? r - 1 : 0) & 1, abort_flag, a.err, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after();
        read_state();
      }
      tc_fence_before();
      named_bar_sync(3, 128);
      if (causal && y == 0) mbar_arrive(bars.s_empty);
      // w -> the operand (pieces of 8 columns; columns dv.. are [z 0 ..])
      const int sb = r % NSOP;
      ok = mbar_wait(&bars.sop_empty[sb], ((r / NSOP) & 1) ^ 1, abort_flag, a.err, kWaitLimitNs);
      if (!ok) break;
      if (has_row) {
        uint8_t* sop = sSOP + sb * SOPT;
#pragma unroll
        for (int q8 = 0; q8 < ACCW / 8; ++q8)
          *reinterpret_cast<uint4*>(sop + (q8 >> 3) * (D * kRowBytes) + sw128_off(row, q8 & 7)) =
              make_uint4(w[4 * q8], w[4 * q8 + 1], w[4 * q8 + 2], w[4 * q8 + 3]);
      }
      fence_proxy_async_smem();
      named_bar_sync(3, 128);
      if (y == 0) mbar_arrive(&bars.sop_full[sb]);
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

// One launch: dense sequences whose blocks fit the K/V ring (every tile is
// loaded once) and whose CTAs are all resident at once (one per SM; the
// launch is cooperative, so it fails rather than run them in waves).  Every
// block must hold at least one chunk: an empty block would publish nothing.
bool block_fused_supported(const FwdLaunch& p, int nb, int num_sms) {
  if (!block_supported(p) || p.cu_seqlens != nullptr || nb < 2) return false;
  const int nc = (p.N + kChunk - 1) / kChunk, bc = block_chunks(p, nb);
  return bc <= NKV && (long long)(nb - 1) * bc < nc &&
         (long long)nb * p.Hkv * p.B <= (long long)num_sms;
}

cudaError_t launch_fwd_bf16_block_fused(const FwdLaunch& p, int nb, float* ws,
                                        cudaStream_t stream) {
  if (ws == nullptr) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_3d(&tq, p.q, D, p.Hq, p.total_tokens, 64) ||
      !make_tmap_3d(&tk, p.k, D, p.Hkv, p.total_tokens, 64) ||
      !make_tmap_3d(&tv, p.v, DV, p.Hkv, p.total_tokens, 64))
    return cudaErrorInvalidValue;
  FusedArgs a;
  a.out = reinterpret_cast<__nv_bfloat16*>(p.out);
  a.cu_seqlens = p.cu_seqlens;
  a.ws = nb > 1 ? ws : nullptr;
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
  // four Q stages (every Q tile of a block is loaded at once), one operand buffer
  using L = Layout<4, 1>;
  auto fk = lt_fused_fwd_kernel<4, 1>;
  cudaError_t e = cudaFuncSetAttribute(fk, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nb, p.Hkv, p.B);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fk, tq, tk, tv, a);
}


}  // namespace lt
