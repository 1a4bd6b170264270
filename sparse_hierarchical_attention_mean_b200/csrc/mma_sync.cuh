// Warp-level tensor-core helpers: mma.sync m16n8k16 (f16/bf16 operands, fp32
// accumulate) and ldmatrix loads of 8x8 b16 tiles, plus the XOR swizzle used
// by the tiles they read.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

namespace dash {

// d (16x8, fp32) += a (16x16, row) * b (16x8, col).  Fragments: a[0..3] hold
// (row gq, k 2tq..), (row gq+8, k 2tq..), (row gq, k 8+2tq..), (row gq+8,
// k 8+2tq..); b0/b1 hold (k 2tq.., col gq) and (k 8+2tq.., col gq); d holds
// (gq, 2tq), (gq, 2tq+1), (gq+8, 2tq), (gq+8, 2tq+1), with gq = lane / 4 and
// tq = lane % 4.
template <typename T>
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  if constexpr (std::is_same<T, __half>::value) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// Four 8x8 b16 tiles; lane i supplies the address of row i % 8 of tile i / 8.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Element offset of (row, col) in a [rows][D] tile of 16-bit values whose
// 16-byte chunks are stored XOR-swizzled by (row & 7): ldmatrix reads of
// eight consecutive rows then hit eight different bank groups.
template <int D>
__device__ __forceinline__ int swz(int row, int col) {
  return row * D + ((((col >> 3) ^ (row & 7))) << 3) + (col & 7);
}

}  // namespace dash
