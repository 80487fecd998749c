// kda_warp_mma.cuh -- warp-level tensor-core products in tf32
// (mma.sync.m16n8k8) and the tf32 high/low split that the backward's and
// the fp32-accuracy forward's tensor-core products (warp-level and tcgen05)
// take.
//
// Fragment layout (lane = 4 g + t, PTX ISA m16n8k8 .tf32): A (16 x 8, row
// major) a0 = (g, t), a1 = (g + 8, t), a2 = (g, t + 4), a3 = (g + 8, t + 4);
// B (8 x 8) b0 = (k = t, n = g), b1 = (k = t + 4, n = g); C / D (16 x 8)
// c0 = (g, 2t), c1 = (g, 2t + 1), c2 = (g + 8, 2t), c3 = (g + 8, 2t + 1).
#pragma once

#include <stdint.h>

namespace kda {

// tf32 with fp32 accuracy: x = hi + lo with hi = x with its 13 low mantissa
// bits cleared (a tf32 value) and lo = x - hi exactly, and
// a b = a_lo b_hi + a_hi b_lo + a_hi b_hi.  A tf32 MMA uses 10 of lo's up to
// 13 significant bits, and the dropped a_lo b_lo is as small, so each
// product's error stays below ~2^-20 of |a b| (two instructions; the tf32
// MMAs of tcgen05 and mma.sync take the same parts).
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = __float_as_uint(x) & 0xFFFFE000u;
  lo = __float_as_uint(x - __uint_as_float(hi));
}

// d += a b
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

}  // namespace kda
