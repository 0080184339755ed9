// Fragment helpers shared by the warp-level-MMA W4A16 kernels.
//
// mma.sync.m16n8k16 with .f16 operands (PTX ISA fragment layout), lane = 4 g + j:
//   A registers {row g, k 2j..2j+1}, {row g+8, k 2j..2j+1},
//               {row g, k 2j+8..2j+9}, {row g+8, k 2j+8..2j+9};
//   B registers {k 2j..2j+1, n g}, {k 2j+8..2j+9, n g};
//   D           {row g, n 2j..2j+1}, {row g+8, n 2j..2j+1}.
// The contraction over k is order-free, so k-slot pairs are mapped to the
// column pairs (e, e+4) of a packed word: the pairs one LOP3 produces.  The
// activations are stored in the same order: each 8-column word's columns as
// (0,4,1,5,2,6,3,7).
#pragma once

#include <stdint.h>

namespace awq {

// Column of position p (0..7) within an 8-column word, in the order above.
__device__ __forceinline__ int frag_perm8(int p) { return (p >> 1) + 4 * (p & 1); }

// (1024 + nibble e, 1024 + nibble e + 4) of a packed word as fp16x2: exact,
// since 1024..1039 are fp16 integers.
__device__ __forceinline__ uint32_t frag_nib2(uint32_t w, int e) {
    return ((w >> (4 * e)) & 0x000F000Fu) | 0x64006400u;
}

__device__ __forceinline__ void frag_mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

}  // namespace awq
