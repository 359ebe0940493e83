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
// resident at once).  For chunk r of block b the state splits into the carry
// of the earlier blocks and the block's own earlier chunks,
//     S_<r = C_b + L_r,   C_b = sum_{b' < b} A_b',   L_r = sum_{r' < r} dS_r',
//     dS_r = phi(K_r)^T [V_r | 1],   A_b = sum_r dS_r,
// so everything but phi(Q_r) C_b is known inside the CTA.  Each CTA
//   1. loads every K/V and Q tile of its block once (all stay resident) and
//      applies phi; accumulates A_b = sum_r dS_r on the tensor cores as soon
//      as the K/V tiles are ready, publishes it to the workspace and arrives
//      at the launch's grid barrier (without waiting);
//   2. keeps the running sums L_1 .. L_{R-1} that the aggregate passes
//      through (parked in accumulator columns that are not yet in use),
//      stages each as a bf16 operand once its K slot is free, and computes
//      per chunk
//          Acc_r = mask(phi(Q_r) phi(K_r)^T) [V_r | 1] + phi(Q_r) [L_r | l_r]
//      (numerator columns and the normaliser column);
//   3. meanwhile waits at the grid barrier, sums the earlier aggregates
//      (causal) or all of them (non-causal) in block order into C_b, and adds
//      phi(Q_r) [C_b | c_b] to each chunk's accumulator as soon as both are
//      ready;
//   4. normalises and stores.
//
// The state accumulator is kept transposed, [V | 1]^T phi(K) (M = 128 value
// columns plus the normaliser row, N = 64 key features), so TMEM lane m holds
// row m of the K-major B operand [S | z]^T of the phi(Q) products.
//
// Warp roles (576 threads; TMEM sub-partition = warp % 4):
//   warps 0-7   transform: phi in place on K and Q tiles (tail rows zeroed);
//               then the grid-barrier wait and the carry sum; then the
//               outputs (warps 0-3 the even items, warps 4-7 the odd ones)
//   warps 8-11  mask: causal mask of the score tile, bf16 in place in TMEM
//   warps 12-15 state: the running sums parked as they pass, the aggregate
//               to the workspace, the grid-barrier arrival, the running sums
//               -> bf16 operands
//   warp 16     TMA producer (every load issued at kernel entry)
//   warp 17     TMEM allocator and MMA issuer (a fixed issue order)
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fwd_common.cuh"
#include "lt_internal.h"
#include "lt_ptx.cuh"

namespace lt {
namespace {
using namespace fwd;

constexpr int D = 64, DV = 64;
constexpr int E = D * DV + D;         // block aggregate: 65 rows of 64 floats
constexpr int E4 = E / 4;             // in float4
constexpr int OPR = DV + 16;          // operand rows: S^T (64), z (1), zeros (15)
constexpr int QT = kChunk * D * 2, KT = kChunk * D * 2, VT = kChunk * DV * 2;
constexpr int KVT = KT + VT;          // one K/V stage: [K][V]
constexpr int ONEST = kChunk * kRowBytes;
constexpr int ACCW = DV + 16;         // accumulator columns: numerator, normaliser, pad
constexpr int NST = 4;                // chunks per block, items per block (max)
static_assert(OPR * kRowBytes <= KT, "a running-sum operand fits a freed K slot");

// TMEM columns: four item accumulators, the score tile, the state
constexpr int TM_ACC = 0, TM_P = NST * ACCW, TM_S = TM_P + kChunk, TM_COLS = 512;
static_assert(TM_S + D <= TM_COLS, "TMEM budget");

struct FusedArgs {
  __nv_bfloat16* out;
  float* ws;        // block aggregates [lane][nb][E] (rows S^T then z)
  int Hq, Hkv, N, G, causal;
  int nb;           // blocks per sequence (lane)
  int bc;           // chunks per block
  float eps;
  int* err;
  // the forward pass continued from a given state (nullptr: zero) and
  // returning the final state (nullptr: not returned), per lane:
  // S [lane][d][dv], z [lane][d] fp32
  const float* s0;
  const float* z0;
  float* s_out;
  float* z_out;
};

constexpr int kThreads = 576;
constexpr int kXf = 256;  // transform threads (warps 0-7, two per SM sub-partition)

struct Layout {
  static constexpr int OFF_Q = 0;                     // item j at j*QT
  static constexpr int OFF_KV = OFF_Q + NST * QT;     // chunk r: [K][V] at r*KVT
  static constexpr int OFF_ONES = OFF_KV + NST * KVT;
  static constexpr int OFF_C = OFF_ONES + ONEST;      // the carry operand
  static constexpr int OFF_BAR = OFF_C + ((OPR * kRowBytes + 1023) & ~1023);
  static constexpr int NBARS = 12 * NST + 2;
  static constexpr int SMEM = OFF_BAR + NBARS * 8 + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
};

// Every barrier completes at most once per launch (phase 0).
struct Bars {
  uint64_t *q_full, *q_xf, *kv_full, *kv_xf;   // per item / chunk: landed, phi applied
  uint64_t *s_full, *s_empty;                  // per chunk r: L_{r+1} in the state; parked
  uint64_t *k_free;                            // per chunk: K slot r's scores are done
  uint64_t *op_full;                           // per chunk r >= 1: L_r staged in K slot r-1
  uint64_t *p_full, *pb_full;                  // per item: score ready; masked bf16 ready
  uint64_t *acc_full;                          // per item: accumulator complete
  uint64_t *agg_full;                          // the aggregate is in the state
  uint64_t *g_arr;                             // the grid-barrier arrival is recorded
  uint64_t *c_full;                            // the carry operand is staged
  uint64_t *drain;                             // issued products complete
};

__device__ __forceinline__ Bars carve(uint8_t* base) {
  uint64_t* b = reinterpret_cast<uint64_t*>(base);
  Bars r;
  r.q_full = b; b += NST;
  r.q_xf = b; b += NST;
  r.kv_full = b; b += NST;
  r.kv_xf = b; b += NST;
  r.s_full = b; b += NST;
  r.s_empty = b; b += NST;
  r.k_free = b; b += NST;
  r.op_full = b; b += NST;
  r.p_full = b; b += NST;
  r.pb_full = b; b += NST;
  r.acc_full = b; b += NST;
  r.agg_full = b++;
  r.g_arr = b++;
  b += NST - 2;  // spare
  r.c_full = b++;
  r.drain = b++;
  return r;
}

// Row `row` of a K-major [OPR x 64] bf16 operand (128-byte swizzle) from 64
// fp32 values: 8 pieces of 16 bytes.
__device__ __forceinline__ void store_operand_row(uint8_t* op, int row, const float (&v)[64]) {
#pragma unroll
  for (int q8 = 0; q8 < 8; ++q8) {
    const uint4 w = make_uint4(pack_bf16x2(v[8 * q8], v[8 * q8 + 1]),
                               pack_bf16x2(v[8 * q8 + 2], v[8 * q8 + 3]),
                               pack_bf16x2(v[8 * q8 + 4], v[8 * q8 + 5]),
                               pack_bf16x2(v[8 * q8 + 6], v[8 * q8 + 7]));
    *reinterpret_cast<uint4*>(op + sw128_off(row, q8)) = w;
  }
}

// The carry C = S0 + the aggregates of blocks [0, nsum) of one lane (base:
// that lane's first aggregate; s0, z0: the lane's given state or nullptr),
// fp32 in block order into acc (PER float4 per thread), rounded once to bf16
// into the K-major operand; rows DV+1 .. OPR-1 zeroed.  Thread u of NT.
template <int NT>
constexpr int gather_per() { return (E4 + NT - 1) / NT; }

template <int NT, int NF>
__device__ __forceinline__ void gather_carry(float4 (&acc)[gather_per<NT>()], const float4* base,
                                             int nsum, uint8_t* op, int u, const float* s0,
                                             const float* z0) {
  constexpr int PER = gather_per<NT>();
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int i = u + e * NT, row = i >> 4, c4 = i & 15;
    acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (s0 != nullptr && i < E4) {
      // aggregate row `row`, entries 4*c4 .. 4*c4+3: column `row` of S (rows
      // 4*c4 .. of the [d][dv] state), or z for row DV
      if (row < DV)
        acc[e] = make_float4(s0[(4 * c4) * DV + row], s0[(4 * c4 + 1) * DV + row],
                             s0[(4 * c4 + 2) * DV + row], s0[(4 * c4 + 3) * DV + row]);
      else
        acc[e] = *reinterpret_cast<const float4*>(z0 + 4 * c4);
    }
  }
#pragma unroll 1
  for (int b0 = 0; b0 < nsum; b0 += NF) {  // NF blocks' loads in flight
    float4 v[NF][PER];
#pragma unroll
    for (int k = 0; k < NF; ++k) {
      if (b0 + k < nsum) {
        const float4* blk = base + (size_t)(b0 + k) * E4;
#pragma unroll
        for (int e = 0; e < PER; ++e)
          if (u + e * NT < E4) v[k][e] = __ldcg(blk + u + e * NT);
      }
    }
#pragma unroll
    for (int k = 0; k < NF; ++k) {
      if (b0 + k < nsum) {
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          acc[e].x += v[k][e].x;
          acc[e].y += v[k][e].y;
          acc[e].z += v[k][e].z;
          acc[e].w += v[k][e].w;
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int i = u + e * NT;
    if (i < E4) {
      const int row = i >> 4, c4 = i & 15;  // 16 float4 per 64-float row
      uint2 w = make_uint2(pack_bf16x2(acc[e].x, acc[e].y), pack_bf16x2(acc[e].z, acc[e].w));
      *reinterpret_cast<uint2*>(op + sw128_off(row, c4 >> 1) + (c4 & 1) * 8) = w;
    }
  }
  // zero rows DV+1 .. OPR-1 (15 rows of 8 pieces)
  for (int i = u; i < (OPR - DV - 1) * 8; i += NT) {
    const int row = DV + 1 + (i >> 3);
    *reinterpret_cast<uint4*>(op + sw128_off(row, i & 7)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// The final state C + base[own] (own < 0: C itself) in fp32, in the [d][dv]
// layout, from gather_carry's acc.
template <int NT>
__device__ __forceinline__ void write_final_state(const float4 (&acc)[gather_per<NT>()],
                                                  const float4* base, int u, float* s_out,
                                                  float* z_out, int own) {
  constexpr int PER = gather_per<NT>();
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int i = u + e * NT;
    if (i < E4) {
      const int row = i >> 4, c4 = i & 15;
      float4 f = acc[e];
      if (own >= 0) {
        const float4 a = __ldcg(base + (size_t)own * E4 + i);
        f.x += a.x;
        f.y += a.y;
        f.z += a.z;
        f.w += a.w;
      }
      if (row < DV) {
        s_out[(4 * c4) * DV + row] = f.x;
        s_out[(4 * c4 + 1) * DV + row] = f.y;
        s_out[(4 * c4 + 2) * DV + row] = f.z;
        s_out[(4 * c4 + 3) * DV + row] = f.w;
      } else {
        *reinterpret_cast<float4*>(z_out + 4 * c4) = f;
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    lt_fused_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_o, const FusedArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  using L = Layout;
  __shared__ volatile int s_abort;
  __shared__ unsigned int s_grid_old;  // the state group's grid-barrier arrival
  __shared__ int s_grid_arrived;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int blk = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  const int t0 = s * a.N, ntok = a.N;
  const int nc = (ntok + kChunk - 1) / kChunk;
  const int c0 = blk * a.bc, c1 = min(c0 + a.bc, nc);
  // the host plans no empty block: every CTA must arrive at the grid barrier
  if (c1 <= c0) return;
  const int Ri = c1 - c0;  // chunks of this block
  const int G = a.G;
  const bool causal = a.causal != 0;
  const int n_items = Ri * G;  // item j: chunk j / G, query head g*G + j % G
  // aggregates in the carry: the earlier blocks (causal) or all (non-causal)
  const int nprev = causal ? blk : a.nb;
  // the final state: the last block, from its carry plus (causal) its own
  // aggregate
  const bool final_state = a.s_out != nullptr && blk + 1 == a.nb;
  const bool publish = !causal || blk + 1 < a.nb || final_state;
  // every block with a carry (earlier blocks or a given state) gathers it
  const bool gath = nprev > 0 || a.s0 != nullptr;
  const size_t lane_idx = (size_t)s * a.Hkv + g;
  const float4* agg_base =
      reinterpret_cast<const float4*>(a.ws) + (size_t)(s * a.Hkv + g) * a.nb * E4;

  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_KV;
  uint8_t* sV = smem + L::OFF_KV + KT;
  uint8_t* sOnes = smem + L::OFF_ONES;
  uint8_t* sC = smem + L::OFF_C;
  Bars bars = carve(smem + L::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + L::NBARS * 8);

  if (tid == 16 * 32) {
    // the producer thread initialises the barriers and issues every tile
    // load before the CTA-wide setup (every tile has its own slot: K/V of
    // every chunk first, the state products need them, then every Q tile);
    // the other threads use the barriers after the barrier below
    s_abort = 0;
    uint64_t* b = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    for (int i = 0; i < L::NBARS; ++i) mbar_init(&b[i], 1);
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_o);
    for (int r = 0; r < Ri; ++r) {
      const int c = c0 + r;
      mbar_arrive_expect_tx(&bars.kv_full[r], KT + VT);
      tma_load_3d(sK + r * KVT, &tm_k, &bars.kv_full[r], 0, g, t0 + c * kChunk);
      tma_load_3d(sV + r * KVT, &tm_v, &bars.kv_full[r], 0, g, t0 + c * kChunk);
    }
    for (int j = 0; j < n_items; ++j) {
      const int r = j / G, h = j % G, c = c0 + r;
      mbar_arrive_expect_tx(&bars.q_full[j], QT);
      tma_load_3d(sQ + j * QT, &tm_q, &bars.q_full[j], 0, g * G + h, t0 + c * kChunk);
    }
  }
  init_ones_block(sOnes, tid, kThreads);
  fence_proxy_async_smem();
  if (warp == 17) tmem_alloc(tmem_slot, TM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_flag = &s_abort;

  // Barrier discipline of the thread groups below: every thread of a group
  // passes the same named barriers in the same order on every path; a failed
  // (bounded) wait only raises the abort flag, and the work after a barrier
  // is skipped while the flag is up.

  // The carry sum, by the transform warps (256 threads) between two
  // barriers 5.
  auto gather_part = [&](int u) {
    float4 acc[gather_per<kXf>()];
    named_bar_sync(5, kXf);
    if (!*abort_flag) {
      gather_carry<kXf, 2>(acc, agg_base, nprev, sC, u,
                           a.s0 ? a.s0 + lane_idx * D * DV : nullptr,
                           a.z0 ? a.z0 + lane_idx * D : nullptr);
      fence_proxy_async_smem();
    }
    named_bar_sync(5, kXf);
    if (u == 0 && !*abort_flag) mbar_arrive(bars.c_full);
    // the final state after the carry is released: off the path to the
    // carry products
    if (final_state && !*abort_flag)
      write_final_state<kXf>(acc, agg_base, u, a.s_out + lane_idx * D * DV,
                             a.z_out + lane_idx * D, causal ? blk : -1);
  };

  // Accumulator of item j -> normalised bf16 row, one thread per row (TMEM
  // lane = chunk row); x in [0, 128) of the group of four warps that passes
  // named barrier `nbar`.  A whole chunk is staged in item j's Q slot (its
  // last reader, the item's final product, is complete) and written by one
  // TMA store; the rows of a ragged last chunk are stored directly (a tile
  // would run into the next sequence).  Returns false once the abort flag is
  // up (read after the group barrier, so the group agrees).
  auto epilogue = [&](int j, int x, int nbar) -> bool {
    const int sp = (x >> 5) & 3, row = x;
    const int r = j / G, h = j % G, c = c0 + r;
    const bool ok = mbar_wait(&bars.acc_full[j], 0, abort_flag, a.err, kWaitLimitNs);
    tc_fence_after();
    uint32_t pk[DV / 2];
    if (ok) {
      const uint32_t t_acc = tmem + TM_ACC + j * ACCW + ((uint32_t)(sp * 32) << 16);
      float n[32];
      const float den = tmem_ld1(t_acc + DV);
      tmem_ld32(t_acc, n);
      tmem_wait_ld();
      const float inv = 1.0f / (den + a.eps);
#pragma unroll
      for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(n[2 * e] * inv, n[2 * e + 1] * inv);
      tmem_ld32(t_acc + 32, n);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) pk[16 + e] = pack_bf16x2(n[2 * e] * inv, n[2 * e + 1] * inv);
    }
    const int valid = min(kChunk, ntok - c * kChunk);
    if (valid == kChunk) {  // uniform over the group
      uint8_t* tile = sQ + j * QT;
      if (ok) {
#pragma unroll
        for (int q = 0; q < DV / 8; ++q)
          *reinterpret_cast<uint4*>(tile + sw128_off(row, q)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
      fence_proxy_async_smem();
      named_bar_sync(nbar, 128);
      if (x == 0 && !*abort_flag) {
        tma_store_3d(&tm_o, tile, 0, g * G + h, t0 + c * kChunk);
        bulk_commit_group();
      }
      return !*abort_flag;
    }
    if (ok && row < valid) {
      uint4* orow = reinterpret_cast<uint4*>(
          a.out + ((size_t)(t0 + c * kChunk + row) * a.Hq + (size_t)(g * G + h)) * DV);
#pragma unroll
      for (int q = 0; q < DV / 8; ++q)
        orow[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    }
    return ok;
  };

  if (warp == 16) {
    // producer: its loads were issued before the setup barrier
    __syncwarp();
  } else if (warp == 17) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_DS = idesc_bf16_f32(kChunk, D, 1, 1);      // [V|1]^T phi(K)
      constexpr uint32_t ID_P = idesc_bf16_f32(kChunk, kChunk, 0, 0);  // phi(Q) phi(K)^T
      constexpr uint32_t ID_PV = idesc_bf16_f32(kChunk, DV + 16, 0, 1);
      constexpr uint32_t ID_QS = idesc_bf16_f32(kChunk, DV + 16, 0, 0);
      const uint64_t dQk = smem_desc_sw128(smem_u32(sQ), 16, 1024);     // K-major phi(Q)
      const uint64_t dKk = smem_desc_sw128(smem_u32(sK), 16, 1024);     // K-major phi(K)
      const uint64_t dKmn = smem_desc_sw128(smem_u32(sK), kBox, 1024);  // MN-major phi(K)
      const uint32_t ones = smem_u32(sOnes);
      // [V | 1] (MN-major; the second 64-element group is the ones block)
      auto vdesc = [&](int r) {
        const uint32_t va = smem_u32(sV) + r * KVT;
        return smem_desc_sw128(va, ones - va, 1024);
      };
      // state (+)= [V_r | 1]^T phi(K_r)
      auto issue_ds = [&](int r, bool accumulate) {
        const uint64_t ad = vdesc(r), bd = desc_advance(dKmn, r * KVT);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          umma_f16_ss(tmem + TM_S, desc_advance(ad, kk * 2048), desc_advance(bd, kk * 2048),
                      ID_DS, (accumulate || kk > 0) ? 1u : 0u);
      };
      // Acc_j (+)= phi(Q_j) Op, Op the K-major [OPR x 64] operand at op
      auto issue_qs = [&](int j, const uint8_t* op, bool accumulate) {
        const uint64_t qa = desc_advance(dQk, j * QT);
        const uint64_t od = smem_desc_sw128(smem_u32(op), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_f16_ss(tmem + TM_ACC + j * ACCW, desc_advance(qa, kk * 32),
                      desc_advance(od, kk * 32), ID_QS, (accumulate || kk > 0) ? 1u : 0u);
      };
      auto issue_score = [&](int j) {
        const int r = j / G;
        const uint64_t qd = desc_advance(dQk, j * QT), kd = desc_advance(dKk, r * KVT);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_f16_ss(tmem + TM_P, desc_advance(qd, kk * 32), desc_advance(kd, kk * 32), ID_P,
                      kk > 0 ? 1u : 0u);
      };
      auto issue_pv = [&](int j) {
        const uint64_t vd = vdesc(j / G);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          umma_f16_ts(tmem + TM_ACC + j * ACCW, tmem + TM_P + kk * 8, desc_advance(vd, kk * 2048),
                      ID_PV, kk > 0 ? 1u : 0u);
      };
      const bool has_carry = gath;
      // A fixed issue order with one blocking (bounded) wait per group: the
      // tensor pipe executes in issue order, so the single score buffer is
      // free again once the previous item's P V has been issued.
      auto W = [&](uint64_t* bar) {
        const bool ok = mbar_wait(bar, 0, abort_flag, a.err, kWaitLimitNs);
        if (ok) tc_fence_after();
        return ok;
      };
      do {
        // 1. the state chunk by chunk (causal: after chunk r it holds
        //    L_{r+1}, which the state warps park before the next product);
        //    after the last chunk it is the block aggregate (what the other
        //    CTAs wait for)
        bool ok = true;
        for (int r = 0; r < Ri && ok; ++r) {
          if (!(ok = W(&bars.kv_xf[r]))) break;
          if (causal && r > 0 && !(ok = W(&bars.s_empty[r - 1]))) break;
          issue_ds(r, r > 0);
          if (causal && r + 1 < Ri) umma_commit(&bars.s_full[r]);
        }
        if (!ok) break;
        umma_commit(bars.agg_full);
        // 2. causal: per item its score, P V (the first item of a chunk after
        //    the chunk's running sum has left its accumulator) and phi(Q) L;
        //    and phi(Q) [C | c] for the items whose local products are
        //    issued, as soon as the carry is staged
        int qc = 0;
        bool c_ready = false;
        auto carry_products = [&](int upto) {
          if (!c_ready) {
            if (!mbar_test(bars.c_full, 0)) return;
            c_ready = true;
            tc_fence_after();
          }
          for (; qc < upto; ++qc) {
            issue_qs(qc, sC, true);
            umma_commit(&bars.acc_full[qc]);
          }
        };
        // item j's products that nothing in the score -> mask -> P V chain
        // waits for: phi(Q) L, then (no carry) the accumulator is complete,
        // or the carry products that are ready
        auto finish = [&](int j) {
          const int r = j / G;
          if (r > 0) {
            if (!W(&bars.op_full[r])) return false;
            issue_qs(j, sK + (r - 1) * KVT, true);
          }
          if (!has_carry)
            umma_commit(&bars.acc_full[j]);
          else
            carry_products(j + 1);
          return true;
        };
        for (int j = 0; j < n_items && causal && ok; ++j) {
          const int r = j / G;
          if (!(ok = W(&bars.q_xf[j]))) break;
          issue_score(j);
          umma_commit(&bars.p_full[j]);
          if (j % G == G - 1) umma_commit(&bars.k_free[r]);
          // the previous item's remaining products run during this mask
          if (j > 0 && !(ok = finish(j - 1))) break;
          if (!(ok = W(&bars.pb_full[j]))) break;
          if (r > 0 && j % G == 0 && !(ok = W(&bars.op_full[r]))) break;
          issue_pv(j);
        }
        if (ok && causal && n_items > 0) ok = finish(n_items - 1);
        if (!ok || !has_carry) break;
        // 3. phi(Q) [C | c] into the remaining accumulators
        if (!c_ready && !W(bars.c_full)) break;
        for (int j = qc; j < n_items; ++j) {
          if (!causal && !W(&bars.q_xf[j])) break;
          issue_qs(j, sC, causal);
          umma_commit(&bars.acc_full[j]);
        }
      } while (false);
      umma_commit(bars.drain);
      int dummy = 0;
      mbar_wait(bars.drain, 0, &dummy, nullptr, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ---------------------------------------------- transform warps
    const int x = tid;  // 0..255
    // every K tile (with V's tail rows zeroed in a ragged chunk), then every Q
    const int T = Ri + n_items;
    for (int t = 0; t < T; ++t) {
      const bool is_kv = t < Ri;
      const int r = t, j = t - Ri;
      mbar_wait(is_kv ? &bars.kv_full[r] : &bars.q_full[j], 0, abort_flag, a.err, kWaitLimitNs);
      if (!*abort_flag) {
        uint8_t* tile = is_kv ? sK + r * KVT : sQ + j * QT;
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
      }
      named_bar_sync(1, kXf);
      if (x == 0 && !*abort_flag) mbar_arrive(is_kv ? &bars.kv_xf[r] : &bars.q_xf[j]);
    }
    if (gath) {
      // the grid barrier (after the state group has arrived), then the carry
      if (x == 0 && mbar_wait(bars.g_arr, 0, abort_flag, a.err, kWaitLimitNs) &&
          s_grid_arrived && (nprev > 0 || final_state))
        grid_wait(s_grid_old, abort_flag, a.err, kWaitLimitNs);
      gather_part(x);
    }
    // the outputs: warps 0-3 the even items, warps 4-7 the odd ones (named
    // barriers 6 and 7); the issuing thread waits for its TMA stores
    bool ok = true;
    for (int j = warp >> 2; j < n_items && ok; j += 2) ok = epilogue(j, x & 127, 6 + (warp >> 2));
    if ((x & 127) == 0) bulk_wait_all();
  } else if (warp < 12) {
    // ---------------------------------------------------- mask warpgroup
    const int x = tid - 256, sp = warp & 3;
    const int row = sp * 32 + lane;  // TMEM lane == chunk row
    // causal mask and bf16 rounding of the score tile, in place in TMEM:
    // fp32 columns [32b, 32b+32) become packed bf16 columns [16b, 16b+16),
    // which only overwrites columns this thread has already read
    for (int j = 0; j < n_items && causal; ++j) {
      mbar_wait(&bars.p_full[j], 0, abort_flag, a.err, kWaitLimitNs);
      tc_fence_after();
      if (!*abort_flag) {
        const uint32_t t_p = tmem + TM_P + ((uint32_t)(sp * 32) << 16);
        // two 32-column blocks per TMEM round trip; fp32 block b becomes
        // packed bf16 block b (columns [16b, 16b+16)), so every store lands
        // on columns that are already read
        auto pack_block = [&](int b, const float (&r)[32], uint32_t (&pk)[16]) {
          if (b < sp) {  // warp-uniform: a block entirely left of the diagonal
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(r[2 * e], r[2 * e + 1]);
          } else if (b == sp) {  // the diagonal block
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float lo = (b * 32 + 2 * e > row) ? 0.0f : r[2 * e];
              const float hi = (b * 32 + 2 * e + 1 > row) ? 0.0f : r[2 * e + 1];
              pk[e] = pack_bf16x2(lo, hi);
            }
          } else {  // right of the diagonal: zero
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = 0u;
          }
        };
#pragma unroll
        for (int b0 = 0; b0 < kChunk / 32; b0 += 2) {
          float ra[32], rb[32];
          uint32_t pk[16];
          if (b0 <= sp) tmem_ld32(t_p + b0 * 32, ra);
          if (b0 + 1 <= sp) tmem_ld32(t_p + (b0 + 1) * 32, rb);
          if (b0 <= sp) tmem_wait_ld();
          pack_block(b0, ra, pk);
          tmem_st16(t_p + b0 * 16, pk);
          pack_block(b0 + 1, rb, pk);
          tmem_st16(t_p + (b0 + 1) * 16, pk);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      named_bar_sync(2, 128);
      if (x == 0 && !*abort_flag) mbar_arrive(&bars.pb_full[j]);
    }
  } else if (warp < 16) {
    // -------------------------------------------------- state warpgroup
    // TMEM state lane m: row m of [S | z]^T (m < 64: column m of S; m = 64:
    // z; 65..127: zero), 64 fp32 columns (key features).  Warps 12-14 cover
    // the operand's 80 rows; warp 15 only joins the barriers.  Thread y == 0
    // does the mbarrier waits for the group.
    const int y = tid - 384, sp = warp & 3;
    const int m = sp * 32 + lane;
    const uint32_t t_s = tmem + TM_S + ((uint32_t)(sp * 32) << 16);
    const bool has_rows = sp < 3;  // warp-uniform
    float v[64];
    auto read_state = [&](uint64_t* full) {
      if (y == 0) mbar_wait(full, 0, abort_flag, a.err, kWaitLimitNs);
      named_bar_sync(3, 128);
      tc_fence_after();
      if (has_rows && !*abort_flag) {
        float* lo = v;
        float* hi = v + 32;
        tmem_ld32(t_s, *reinterpret_cast<float(*)[32]>(lo));
        tmem_ld32(t_s + 32, *reinterpret_cast<float(*)[32]>(hi));
        tmem_wait_ld();
      }
      tc_fence_before();
      named_bar_sync(3, 128);
    };
    // 1. causal: the running sums L_1 .. L_{Ri-1} as the state passes
    //    through them, each parked in the accumulator columns of the first
    //    item of its chunk (unused until that item's P V)
    for (int r = 0; r + 1 < Ri && causal; ++r) {
      read_state(&bars.s_full[r]);
      if (y == 0 && !*abort_flag) mbar_arrive(&bars.s_empty[r]);
      if (has_rows && !*abort_flag) {
        const uint32_t t_park = tmem + TM_ACC + (r + 1) * G * ACCW + ((uint32_t)(sp * 32) << 16);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t bits[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) bits[e] = __float_as_uint(v[16 * q4 + e]);
          tmem_st16(t_park + 16 * q4, bits);
        }
        tmem_wait_st();
      }
    }
    // 2. the block aggregate: publish, arrive at the grid barrier (every CTA
    //    exactly once, on every path).  The group barrier orders every
    //    thread's aggregate writes before the arriving thread's release at
    //    gpu scope (release is cumulative).
    read_state(bars.agg_full);
    if (publish && has_rows && m <= DV && !*abort_flag) {
      float4* dst = reinterpret_cast<float4*>(
          a.ws + (((size_t)(s * a.Hkv + g) * a.nb + blk) * E + (size_t)m * D));
#pragma unroll
      for (int u = 0; u < 16; ++u)
        dst[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
    }
    named_bar_sync(3, 128);
    if (y == 0) {
      // the transform group waits at the barrier
      unsigned int grid_old = 0;
      const bool arrived = grid_arrive(&grid_old, abort_flag, a.err);
      s_grid_old = grid_old;
      s_grid_arrived = arrived ? 1 : 0;
      mbar_arrive(bars.g_arr);
    }
    // 3. causal: each parked running sum L_r, staged into the K slot of the
    //    chunk before once that slot's scores are done (this frees its
    //    accumulator columns for P V)
    for (int r = 1; r < Ri && causal; ++r) {
      if (y == 0) mbar_wait(&bars.k_free[r - 1], 0, abort_flag, a.err, kWaitLimitNs);
      named_bar_sync(3, 128);
      tc_fence_after();
      if (has_rows && !*abort_flag) {
        const uint32_t t_park = tmem + TM_ACC + r * G * ACCW + ((uint32_t)(sp * 32) << 16);
        tmem_ld32(t_park, *reinterpret_cast<float(*)[32]>(v));
        tmem_ld32(t_park + 32, *reinterpret_cast<float(*)[32]>(v + 32));
        tmem_wait_ld();
        if (m < OPR) store_operand_row(sK + (r - 1) * KVT, m, v);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(3, 128);
      if (y == 0 && !*abort_flag) mbar_arrive(&bars.op_full[r]);
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

// One launch: dense sequences whose blocks fit the K/V slots (every tile is
// loaded once) with at most four (chunk, query head) items per block, and
// whose CTAs are all resident at once (one per SM; the launch is
// cooperative, so it fails rather than run them in waves).  Every block must
// hold at least one chunk: an empty block would publish nothing.
bool block_fused_supported(const FwdLaunch& p, int nb, int num_sms) {
  if (!block_supported(p) || p.cu_seqlens != nullptr || nb < 2) return false;
  const int nc = (p.N + kChunk - 1) / kChunk, bc = block_chunks(p, nb);
  const int G = p.Hq / p.Hkv;
  return bc * G <= NST && (long long)(nb - 1) * bc < nc &&
         (long long)nb * p.Hkv * p.B <= (long long)num_sms;
}

cudaError_t launch_fwd_bf16_block_fused(const FwdLaunch& p, int nb, float* ws,
                                        cudaStream_t stream) {
  return launch_fwd_bf16_block_fused_state(p, nb, ws, nullptr, nullptr, nullptr, nullptr,
                                           stream);
}

cudaError_t launch_fwd_bf16_block_fused_state(const FwdLaunch& p, int nb, float* ws,
                                              const float* s0, const float* z0, float* s_out,
                                              float* z_out, cudaStream_t stream) {
  if (ws == nullptr) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_3d(&tq, p.q, D, p.Hq, p.total_tokens, 64) ||
      !make_tmap_3d(&tk, p.k, D, p.Hkv, p.total_tokens, 64) ||
      !make_tmap_3d(&tv, p.v, DV, p.Hkv, p.total_tokens, 64) ||
      !make_tmap_3d(&to, p.out, DV, p.Hq, p.total_tokens, 64))
    return cudaErrorInvalidValue;
  FusedArgs a;
  a.out = reinterpret_cast<__nv_bfloat16*>(p.out);
  a.ws = ws;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.N = p.N;
  a.G = p.Hq / p.Hkv;
  a.causal = p.causal;
  a.nb = nb;
  a.bc = block_chunks(p, nb);
  a.eps = p.eps;
  a.err = p.err;
  a.s0 = s0;
  a.z0 = z0;
  a.s_out = s_out;
  a.z_out = z_out;
  auto fk = lt_fused_fwd_kernel;
  cudaError_t e =
      cudaFuncSetAttribute(fk, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nb, p.Hkv, p.B);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Layout::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fk, tq, tk, tv, to, a);
}

}  // namespace lt
