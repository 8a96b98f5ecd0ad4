// mma.cuh -- warp-level tensor-core primitives (mma.sync, ldmatrix) used by
// the decode kernel's per-block arithmetic on sm_100a.
//
// Fragment layouts (PTX ISA, "Matrix fragments for mma.m16n8k*"): lane =
// 4 * g + t (g = groupID 0..7, t = thread-in-group 0..3).
//   8-bit  m16n8k32  A (row): a0 = A[g][4t..4t+3], a1 = A[g+8][4t..4t+3],
//                             a2 = A[g][16+4t..], a3 = A[g+8][16+4t..]
//                    B (col): b0 = B[4t..4t+3][g], b1 = B[16+4t..16+4t+3][g]
//   8-bit  m16n8k16  A: a0 = A[g][4t..4t+3], a1 = A[g+8][4t..4t+3];
//                    B: b0 = B[4t..4t+3][g]
//   f16    m16n8k16  A: a0 = A[g][2t,2t+1], a1 = A[g+8][2t,2t+1],
//                       a2 = A[g][2t+8,2t+9], a3 = A[g+8][2t+8,2t+9];
//                    B: b0 = B[2t,2t+1][g], b1 = B[2t+8,2t+9][g]
//   f16    m16n8k8   A: a0 = A[g][2t,2t+1], a1 = A[g+8][2t,2t+1]; B: b0 = B[2t,2t+1][g]
//   C/D (all): c0 = C[g][2t], c1 = C[g][2t+1], c2 = C[g+8][2t], c3 = C[g+8][2t+1]
#pragma once

#include <cstdint>

namespace hyb {

// D = A * B + C, s8 x s8 -> s32, m16n8k32
__device__ __forceinline__ void mma_s8s8_k32(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B, s8 (A) x u8 (B) -> s32, m16n8k16, zero accumulator in
__device__ __forceinline__ void mma_s8u8_k16_z(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm("mma.sync.aligned.m16n8k16.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%7,%7,%7};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(b0), "r"(0));
}

// D = A * B + C, f16 x f16 -> f32, m16n8k16
__device__ __forceinline__ void mma_f16_k16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B, f16 x f16 -> f32, m16n8k8, zero accumulator in
__device__ __forceinline__ void mma_f16_k8_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  const float z = 0.f;
  asm("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%7,%7,%7};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0), "f"(z));
}

// Four 8x8 matrices of 16-bit elements (or 8 rows x 16 bytes): lane L gives
// the shared address of row L % 8 of matrix L / 8; register m receives lane
// (g, t)'s piece of matrix m: row g, bytes 4t..4t+3.
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}

// As ldmatrix_x4, transposed: register m of lane (g, t) holds elements
// (row 2t, column g) and (row 2t + 1, column g) of matrix m (16-bit each).
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}

// Byte permute (PTX prmt.b32): result byte i = byte sel[4i+3:4i] of {b, a}.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

}  // namespace hyb
