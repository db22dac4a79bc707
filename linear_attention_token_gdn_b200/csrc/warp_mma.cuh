// warp_mma.cuh -- warp-synchronous tensor-core products (mma.sync m16n8k16, fp16 operands, fp32
// accumulation) on fp32 data held in shared memory, with each fp32 operand entered as a
// rounded fp16 high part plus its fp16 remainder: hi*hi + hi*lo + lo*hi keeps about 21
// significant bits, so a product of fp32 matrices comes out at nearly fp32 accuracy.  Used for
// the small block products of the chunk's triangular inverse, where latency (about 20 cycles
// per dependent mma.sync, measured) matters more than throughput.
//
// Fragment layouts of mma.sync.m16n8k16 (PTX ISA, "Matrix fragments for mma.m16n8k16"), with
// g = lane / 4 and t = lane % 4:
//   A 16x16 row-major: reg0 = A[g][2t..2t+1], reg1 = A[g+8][2t..2t+1], reg2 = A[g][2t+8..2t+9],
//                      reg3 = A[g+8][2t+8..2t+9]
//   B 16x8:            reg0 = B[2t..2t+1][g],  reg1 = B[2t+8..2t+9][g]
//   C 16x8:            c0, c1 = C[g][2t..2t+1],  c2, c3 = C[g+8][2t..2t+1]
// The element with the lower index sits in the low half of each 32-bit register.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

namespace gdn {
namespace wm {

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// The same shape with bf16 operands (BF) or fp16 operands.
template <bool BF>
__device__ __forceinline__ void mma16816x(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (BF) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}

// Four 8x8 16-bit matrices from shared memory (ldmatrix): lanes 8i .. 8i+7 give the row addresses
// of matrix i, register i receives it in the fragment layout (row lane / 4, columns 2 (lane % 4),
// +1).  The .trans form delivers each matrix transposed (column lane / 4, rows 2 (lane % 4), +1).
__device__ __forceinline__ void ldsm_x4(uint32_t saddr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t saddr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr)
                 : "memory");
}

// A pair of bf16 values as a pair of fp16 values, each rounded to nearest (exact for 2^-14 <= |x|
// < 65504): bf16 is the top half of an fp32 word.
__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t x) {
    const __half2 h = __floats2half2_rn(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
    return *reinterpret_cast<const uint32_t*>(&h);
}

// (x0, x1) -> fp16 pairs hi = round(x), lo = round(x - hi)
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(x0, x1);
    const float2 f = __half22float2(h);
    const __half2 l = __floats2half2_rn(x0 - f.x, x1 - f.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// A fragment of the 16x16 tile at (r0, c0) of an fp32 matrix with row stride ld, times `scale`.
__device__ __forceinline__ void load_a(const float* m, int ld, int r0, int c0, float scale, uint32_t (&hi)[4],
                                       uint32_t (&lo)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + g + 8 * (i & 1), c = c0 + 2 * t + 8 * (i >> 1);
        const float2 v = *reinterpret_cast<const float2*>(m + r * ld + c);
        split2(scale * v.x, scale * v.y, hi[i], lo[i]);
    }
}

// B fragment of the 16x8 tile at (r0 = k, c0 = n) of an fp32 matrix with row stride ld.
__device__ __forceinline__ void load_b(const float* m, int ld, int r0, int c0, uint32_t (&hi)[2], uint32_t (&lo)[2]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = r0 + 2 * t + 8 * i, c = c0 + g;
        split2(m[r * ld + c], m[(r + 1) * ld + c], hi[i], lo[i]);
    }
}

// d += A * B with both operands split: three mma.sync.
__device__ __forceinline__ void mma_split(float (&d)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4],
                                          const uint32_t (&bh)[2], const uint32_t (&bl)[2]) {
    mma16816(d, al, bh);
    mma16816(d, ah, bl);
    mma16816(d, ah, bh);
}

// The 16x8 C tile at (r0, c0) of an fp32 matrix with row stride ld.
__device__ __forceinline__ void store_c(float* m, int ld, int r0, int c0, const float (&d)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2*>(m + (r0 + g) * ld + c0 + 2 * t) = make_float2(d[0], d[1]);
    *reinterpret_cast<float2*>(m + (r0 + g + 8) * ld + c0 + 2 * t) = make_float2(d[2], d[3]);
}

}  // namespace wm
}  // namespace gdn
