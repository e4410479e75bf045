// fused_tc.cuh -- register-fragment tensor-core pieces of the persistent layer
// kernel at 2..8 tokens: NVFP4 rows decoded in registers straight into the A
// fragments of mma.sync m16n8k16 (f16 x f16 -> f32), activations as the B
// fragments (8 columns = the expert's tokens), read with ldmatrix.
//
// K mapping. The m16n8k16 A fragment gives lane (g, t) two k pairs per row:
// logical k (2t, 2t+1) and (2t+8, 2t+9). Contraction order is free, so a lane
// instead takes 32 consecutive elements of a 128-element K segment from one
// 16-byte code chunk (elements 32t .. 32t+31, i.e. blocks 2t and 2t+1 of the
// segment's eight 16-element scale blocks), and MMA j (j = 0..7) of the
// segment uses code bytes 2j (as logical k 2t, 2t+1) and 2j+1 (as 2t+8, 2t+9):
// physical elements 32t+4j+{0,1} and 32t+4j+{2,3}. The B operand (x or h) is
// stored in shared memory in exactly that order, so one ldmatrix.x4 yields
// the b0/b1 registers of two MMAs (see tc_b_offset).
//
// Exactness. An E2M1 value times its E4M3 block scale has at most 6
// significant bits and lies in [2^-10, 2688], so the scaled weight is exact in
// f16; the MMA multiplies exactly and accumulates in f32. The activations are
// the same f16 values (x or h times a power of two) the CUDA-core loops use.
#pragma once

#include "common.cuh"

namespace flint {

constexpr int kTcStageK = 512;          // K elements per gate/up stage
constexpr int kTcStageCodes = 16 * 256; // 16 rows x 256 code bytes (two 128-byte swizzled boxes)
constexpr int kTcStageScales = 16 * 32; // 16 rows x 32 scale bytes
constexpr int kTcUnits = 8;             // gate/up units per 16-row tile

// mma.sync m16n8k16, A row-major f16, B column-major f16, f32 accumulate.
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 8x8 b16 matrices; lane l supplies the row address of matrix l/8, row l%8.
__device__ __forceinline__ void ldsm_x4(const void* p, uint32_t& d0, uint32_t& d1, uint32_t& d2, uint32_t& d3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(d0), "=r"(d1), "=r"(d2), "=r"(d3)
               : "r"(smem_addr(p)));
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Byte offset, within a row of the B operand, of element k: segment k/128
// holds 16 matrices of 16 bytes; matrix 2j+h, column 2t+e holds the element
// 32t + 4j + 2h + e of the segment.
__host__ __device__ __forceinline__ int tc_b_offset(int k) {
  const int r = k & 127, t = r >> 5, w = r & 31;
  return (k >> 7) * 256 + (w >> 1) * 16 + (2 * t + (w & 1)) * 2;
}

// Row stride (bytes) of a B-operand row of K elements: padded by 16 bytes so
// the eight rows of an ldmatrix fall in distinct bank groups.
__host__ __device__ constexpr int tc_b_stride(int K) { return 2 * K + 16; }

// One 128-element K segment of a 16-row tile: row g from the 16-byte code
// chunk ra with its two scale bytes sa2 (blocks 2t, 2t+1; low byte first), row
// g+8 from rb / sb2; b[2j], b[2j+1] the B registers of MMA j. Even and odd
// MMAs accumulate into c0 and c1 (two dependency chains of four); the caller
// adds c1 to c0 once, in a fixed order.
__device__ __forceinline__ void tc_segment(float (&c0)[4], float (&c1)[4], const uint4 ra, const uint4 rb, uint32_t sa2,
                                           uint32_t sb2, const uint32_t (&b)[16]) {
  uint32_t ha, hb;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(ha) : "h"(static_cast<uint16_t>(sa2)));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hb) : "h"(static_cast<uint16_t>(sb2)));
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t sa = __byte_perm(ha, 0, half ? 0x3232 : 0x1010);
    const uint32_t sb = __byte_perm(hb, 0, half ? 0x3232 : 0x1010);
    uint32_t qa[8], qb[8];
    e2m1x8_to_f16x2(half ? ra.z : ra.x, *reinterpret_cast<uint32_t(*)[4]>(&qa[0]));
    e2m1x8_to_f16x2(half ? ra.w : ra.y, *reinterpret_cast<uint32_t(*)[4]>(&qa[4]));
    e2m1x8_to_f16x2(half ? rb.z : rb.x, *reinterpret_cast<uint32_t(*)[4]>(&qb[0]));
    e2m1x8_to_f16x2(half ? rb.w : rb.y, *reinterpret_cast<uint32_t(*)[4]>(&qb[4]));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      qa[i] = hmul2_u32(qa[i], sa);
      qb[i] = hmul2_u32(qb[i], sb);
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = 4 * half + jj;
      mma16816((jj & 1) ? c1 : c0, qa[2 * jj], qb[2 * jj], qa[2 * jj + 1], qb[2 * jj + 1], b[2 * j], b[2 * j + 1]);
    }
  }
}

// The B registers of one segment: four ldmatrix.x4 from the lane's row base
// (the row of column lane%8) at segment byte offset `seg_off`.
__device__ __forceinline__ void tc_load_b(const uint8_t* row_base, int seg_off, int lane, uint32_t (&b)[16]) {
  const uint8_t* p = row_base + seg_off + (lane >> 3) * 16;
#pragma unroll
  for (int q = 0; q < 4; ++q) ldsm_x4(p + q * 64, b[4 * q], b[4 * q + 1], b[4 * q + 2], b[4 * q + 3]);
}

// Gate/up tile row order: MMA row g is the gate row of unit pi(g) and row g+8
// its up row, pi = (0 2 1 3 4 6 5 7). With the 128-byte swizzle (16-byte chunk
// index XOR row % 8) the two rows one load phase reads then sit in opposite
// halves of the bank space.
__device__ __forceinline__ int tc_unit_of(int g) { return (g & 4) | ((g & 1) << 1) | ((g >> 1) & 1); }

// Address of the 16-byte code chunk of tile row `row` (0..15), segment `seg`
// (0..3) of a gate/up stage, lane column t: stage = two swizzled boxes of
// 16 rows x 128 bytes.
__device__ __forceinline__ const uint8_t* tc_code_chunk(const uint8_t* stage, int row, int seg, int t) {
  const int chunk = (((seg & 1) << 2) | t) ^ (row & 7);
  return stage + (seg >> 1) * 2048 + row * 128 + (chunk << 4);
}

}  // namespace flint
