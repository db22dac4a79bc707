// common.cuh -- shared device helpers of libgdn (dtype conversion, reductions,
// sequence lookup, the device error word).  Included once, by gdn_lib.cu.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

enum Dtype : int { kF32 = 0, kBF16 = 1, kF16 = 2 };

// Bits of the device error word (read and cleared by gdn_check_device_error).
enum ErrBits : unsigned {
    kErrTimeout = 1u,      // a bounded wait ran out
    kErrSeqlens = 2u,      // cu_seqlens not non-decreasing / out of [0, N]
    kErrSlot = 4u,         // a decode row named a state slot out of range
    kErrBounds = 8u,       // bounds-checking build: a computed global index fell outside its tensor
};

__device__ unsigned int g_error_word;

__device__ __forceinline__ void raise_error(unsigned bits) { atomicOr(&g_error_word, bits); }

// The bounds-checking build (compiled with -DGDN_BOUNDS_CHECK into libgdn_debug.so) tests the
// computed global indices of the kernels against their tensors' extents: in_bounds(i, n) is
// 0 <= i < n, and otherwise flags kErrBounds so that the caller skips the access.  In the
// release build every check is the constant true.
__device__ __forceinline__ bool in_bounds(long long i, long long n) {
#ifdef GDN_BOUNDS_CHECK
    if (i < 0 || i >= n) {
        raise_error(kErrBounds);
        return false;
    }
#else
    (void)i;
    (void)n;
#endif
    return true;
}

// ---- scalar / vector loads and stores in any of the three element types -------------

__device__ __forceinline__ float ld1(const void* p, int dt, size_t i) {
    if (dt == kF32) return reinterpret_cast<const float*>(p)[i];
    if (dt == kBF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    return __half2float(reinterpret_cast<const __half*>(p)[i]);
}

__device__ __forceinline__ void st1(void* p, int dt, size_t i, float x) {
    if (dt == kF32) reinterpret_cast<float*>(p)[i] = x;
    else if (dt == kBF16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
    else reinterpret_cast<__half*>(p)[i] = __float2half_rn(x);
}

// Four consecutive elements starting at element i (i a multiple of 4; 8- or 16-byte load).
__device__ __forceinline__ float4 ld4(const void* p, int dt, size_t i) {
    if (dt == kF32) return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
    uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const char*>(p) + 2 * i);
    float4 r;
    if (dt == kBF16) {
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
        float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
        r = make_float4(fa.x, fa.y, fb.x, fb.y);
    } else {
        __half2 a = *reinterpret_cast<__half2*>(&u.x);
        __half2 b = *reinterpret_cast<__half2*>(&u.y);
        float2 fa = __half22float2(a), fb = __half22float2(b);
        r = make_float4(fa.x, fa.y, fb.x, fb.y);
    }
    return r;
}

__device__ __forceinline__ void st4(void* p, int dt, size_t i, float4 x) {
    if (dt == kF32) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + i) = x;
        return;
    }
    uint2 u;
    if (dt == kBF16) {
        __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y), b = __floats2bfloat162_rn(x.z, x.w);
        u.x = *reinterpret_cast<uint32_t*>(&a);
        u.y = *reinterpret_cast<uint32_t*>(&b);
    } else {
        __half2 a = __floats2half2_rn(x.x, x.y), b = __floats2half2_rn(x.z, x.w);
        u.x = *reinterpret_cast<uint32_t*>(&a);
        u.y = *reinterpret_cast<uint32_t*>(&b);
    }
    *reinterpret_cast<uint2*>(reinterpret_cast<char*>(p) + 2 * i) = u;
}

// 16-bit operands in the input's own format (bf16 or fp16), rounded to nearest.
template <bool BF>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    if constexpr (BF) {
        __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&v);
    } else {
        __half2 v = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&v);
    }
}

template <bool BF>
__device__ __forceinline__ float2 unpack2(uint32_t u) {
    if constexpr (BF) {
        return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
    } else {
        return __half22float2(*reinterpret_cast<__half2*>(&u));
    }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + __expf(-x)); }

// softplus(x) = log(1 + e^x) in the overflow-free form max(x,0) + log1p(e^-|x|).
__device__ __forceinline__ float softplusf_(float x) { return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x))); }

// Bounds [start, end) of sequence n; cu == NULL means equal lengths L = N / num_seqs.
// Out-of-range or decreasing offsets are clamped (an empty range) and flagged.
__device__ __forceinline__ void seq_bounds(const int32_t* cu, int n, int num_seqs, int N, int& start,
                                           int& end) {
    if (cu == nullptr) {
        int L = N / num_seqs;
        start = n * L;
        end = start + L;
        return;
    }
    int a = cu[n], b = cu[n + 1];
    if (a < 0 || b < a || b > N) {
        raise_error(kErrSeqlens);
        a = min(max(a, 0), N);
        b = max(a, min(b, N));
    }
    start = a;
    end = b;
}

// Sequence start of token t (binary search over cu_seqlens); -1 when t lies past the last
// sequence.  cu == NULL: equal lengths.
__device__ __forceinline__ int seq_start_of(const int32_t* cu, int num_seqs, int N, int t) {
    if (cu == nullptr) {
        int L = N / num_seqs;
        return L > 0 ? (t / L) * L : 0;
    }
    if (t >= cu[num_seqs]) return -1;
    int lo = 0, hi = num_seqs - 1;  // find the last n with cu[n] <= t
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    return cu[lo];
}

}  // namespace gdn
