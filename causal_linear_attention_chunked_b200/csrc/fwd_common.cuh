// fwd_common.cuh -- pieces shared by the bf16 forward kernels: chunk
// geometry, the in-place feature-map transform of TMA-loaded tiles, the
// 128-byte swizzle addressing, the normaliser operand block, kernel
// arguments and the host-side tensor-map encoder.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lt_ptx.cuh"

namespace lt {
namespace fwd {

constexpr int kChunk = 128;          // tokens per chunk (MMA M for the row tiles)
constexpr int kRowBytes = 128;       // one swizzle atom row: 64 bf16
constexpr int kBox = kChunk * kRowBytes;  // one 64-column box of a chunk tile
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait

// phi in place over a [kChunk x (NBOX*64)] bf16 tile (rows of 128-byte
// boxes, swizzled; phi is elementwise so the swizzle does not matter).
// Rows >= valid are zeroed.  NT threads (tid in [0, NT)).
// Without apply_phi the rows below `valid` are only converted to the bf16
// operand type (nothing to do for bf16 inputs).
template <int NBOX, int NT = 128, class VAR = VarDefault>
__device__ __forceinline__ void xf_tile(uint8_t* tile, int valid, bool apply_phi, int tid) {
  constexpr int kChunks = kChunk * NBOX * 8;  // 16-byte pieces
#pragma unroll 4
  for (int ch = tid; ch < kChunks; ch += NT) {
    const int rem = ch % (kChunk * 8);
    const int row = rem >> 3;
    uint4* p = reinterpret_cast<uint4*>(tile + (ch / (kChunk * 8)) * kBox + rem * 16);
    uint4 v = *p;
    if (row >= valid) {
      v = make_uint4(0u, 0u, 0u, 0u);
    } else if (apply_phi) {
      v.x = phi2<VAR>(v.x);
      v.y = phi2<VAR>(v.y);
      v.z = phi2<VAR>(v.z);
      v.w = phi2<VAR>(v.w);
    } else if (VAR::kIn != kInBf16) {
      v.x = conv2<VAR>(v.x);
      v.y = conv2<VAR>(v.y);
      v.z = conv2<VAR>(v.z);
      v.w = conv2<VAR>(v.w);
    } else {
      continue;
    }
    *p = v;
  }
}

// phi in place over a full [kChunk x (NBOX*64)] bf16 tile (every row
// valid).  The NBOX boxes are contiguous, so thread t takes the 16-byte
// pieces t, t + NT, ...; all loads are issued before the arithmetic.
template <int NBOX, int NT, class VAR = VarDefault>
__device__ __forceinline__ void phi_tile_full(uint8_t* tile, int tid) {
  constexpr int kPieces = kChunk * NBOX * 8;
  constexpr int kIt = (kPieces + NT - 1) / NT;
  constexpr bool kRagged = kPieces % NT != 0;  // the last round covers part of the threads
  uint4* p = reinterpret_cast<uint4*>(tile) + tid;
  const bool last = !kRagged || tid + (kIt - 1) * NT < kPieces;
  uint4 v[kIt];
#pragma unroll
  for (int i = 0; i < kIt; ++i)
    if (i < kIt - 1 || last) v[i] = p[i * NT];
#pragma unroll
  for (int i = 0; i < kIt; ++i) {
    v[i].x = phi2<VAR>(v[i].x);
    v[i].y = phi2<VAR>(v[i].y);
    v[i].z = phi2<VAR>(v[i].z);
    v[i].w = phi2<VAR>(v[i].w);
  }
#pragma unroll
  for (int i = 0; i < kIt; ++i)
    if (i < kIt - 1 || last) p[i * NT] = v[i];
}

// phi (apply_phi) and zeroing of the rows >= valid: the fast path for full
// tiles, the general loop for the ragged last chunk.
template <int NBOX, int NT, class VAR = VarDefault>
__device__ __forceinline__ void prep_tile(uint8_t* tile, int valid, bool apply_phi, int tid) {
  if (valid >= kChunk) {
    if (apply_phi) phi_tile_full<NBOX, NT, VAR>(tile, tid);
  } else {
    xf_tile<NBOX, NT, VAR>(tile, valid, apply_phi, tid);
  }
}

// Byte offset of the 16-byte piece holding columns [8*jj, 8*jj+8) of row
// `row` inside a 128-byte-swizzled 64-column box (1024-byte aligned).
__device__ __forceinline__ uint32_t sw128_off(int row, int jj) {
  return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((jj ^ (row & 7)) << 4));
}

struct FwdArgs {
  __nv_bfloat16* out;
  const int32_t* cu_seqlens;
  const float* ws;  // block aggregates [sequence][KV head][nb][d*dv + d], or nullptr
  int B, Hq, Hkv, N, G, causal;
  int nb;  // blocks per sequence
  int bc;  // chunks per block
  float eps;
  int total_tokens;
  int* err;
};

// The [1 | 0 ... 0] block: the extra B operand whose products give the
// normaliser (phi(K)^T 1 and the row sums of the masked scores).  Row r
// holds bf16 1.0 in logical column 0, zeros elsewhere (128-byte swizzle).
__device__ __forceinline__ void init_ones_block(uint8_t* ones, int tid, int nthreads) {
  for (int ch = tid; ch < kChunk * 8; ch += nthreads) {
    const int row = ch >> 3, phys = ch & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (phys == (row & 7)) v.x = 0x3F80u;  // logical piece 0 lands at (0 ^ row%8)
    *reinterpret_cast<uint4*>(ones + row * kRowBytes + phys * 16) = v;
  }
}

// host side
inline bool make_tmap_3d(CUtensorMap* m, const void* base, int inner, int heads, long long tokens,
                  int box_inner, bool f16 = false) {
  using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    encode = reinterpret_cast<EncodeFn>(fn);
  }
  const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)heads, (cuuint64_t)tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * heads * 2};
  const cuuint32_t box[3] = {(cuuint32_t)box_inner, 1u, (cuuint32_t)kChunk};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapDataType type =
      f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return encode(m, type, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dense [B][N][heads][inner] bf16 tensor as a 4-D map (inner, head, token in
// the sequence, sequence) with a {box_inner, 1, kChunk, 1} box: a tile
// stored at the end of a sequence is clipped at N instead of running into
// the next sequence.
inline bool make_tmap_4d_dense(CUtensorMap* m, const void* base, int inner, int heads, long long n,
                               long long b, int box_inner) {
  using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    encode = reinterpret_cast<EncodeFn>(fn);
  }
  const cuuint64_t row = (cuuint64_t)inner * heads * 2;
  const cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)heads, (cuuint64_t)n, (cuuint64_t)b};
  const cuuint64_t strides[3] = {(cuuint64_t)inner * 2, row, row * (cuuint64_t)n};
  const cuuint32_t box[4] = {(cuuint32_t)box_inner, 1u, (cuuint32_t)kChunk, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace fwd
}  // namespace lt
