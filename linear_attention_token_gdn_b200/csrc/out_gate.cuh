// out_gate.cuh -- eq. (11) of "On the design of Qwen3.8-Next architecture", section 2.1.1,
// without the output projection W_o: out = sigmoid(z) * y / sqrt(mean(y^2) + eps) * (1 + w),
// the zero-centred RMSNorm over dv per (token, head) followed by the sigmoid output gate.
// HBM-bound elementwise work.  The storage types are template parameters, so every load is a
// straight-line 16-byte vector access: a lane owns PER adjacent channels (4 when y, z and out
// are all fp32, else 8), DV / PER lanes share a row, and a warp covers 32 / (DV / PER) rows per
// pass and kGateRows passes (half as many with 8 channels); every row's y and z are loaded
// before the reductions, which interleave.
#pragma once
#include "common.cuh"

namespace gdn {

constexpr int kGateWarps = 8;
constexpr int kGateRows = 4;  // passes per warp with 4 channels per lane (2 with 8)

// PER consecutive elements of storage type DT starting at element i (16-byte aligned).
template <int DT, int PER>
__device__ __forceinline__ void ldv(const void* p, size_t i, float (&x)[PER]) {
    if constexpr (DT == kF32) {
#pragma unroll
        for (int q = 0; q < PER / 4; ++q) {
            const float4 v = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i)[q];
            x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
        }
    } else if constexpr (PER == 4) {
        const uint2 v = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(p) + i);
        const float2 a = unpack2<DT == kBF16>(v.x), b = unpack2<DT == kBF16>(v.y);
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
#pragma unroll
        for (int q = 0; q < PER / 8; ++q) {
            const uint4 v = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p) + i)[q];
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = unpack2<DT == kBF16>(w4[e]);
                x[8 * q + 2 * e] = f.x;
                x[8 * q + 2 * e + 1] = f.y;
            }
        }
    }
}

template <int DT, int PER>
__device__ __forceinline__ void stv(void* p, size_t i, const float (&x)[PER]) {
    if constexpr (DT == kF32) {
#pragma unroll
        for (int q = 0; q < PER / 4; ++q)
            reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + i)[q] =
                make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
    } else if constexpr (PER == 4) {
        *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p) + i) =
            make_uint2(pack2<DT == kBF16>(x[0], x[1]), pack2<DT == kBF16>(x[2], x[3]));
    } else {
#pragma unroll
        for (int q = 0; q < PER / 8; ++q)
            reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p) + i)[q] = make_uint4(
                pack2<DT == kBF16>(x[8 * q], x[8 * q + 1]), pack2<DT == kBF16>(x[8 * q + 2], x[8 * q + 3]),
                pack2<DT == kBF16>(x[8 * q + 4], x[8 * q + 5]), pack2<DT == kBF16>(x[8 * q + 6], x[8 * q + 7]));
    }
}

template <int DV, int YT, int ZT>
struct GateShape {
    static constexpr int PER0 = (YT == kF32 && ZT == kF32) ? 4 : 8;
    static constexpr int PER = PER0 < DV ? PER0 : DV;  // channels per lane
    static constexpr int LPR = DV / PER;                // lanes per row
    static constexpr int RPP = 32 / LPR;                // rows per warp pass
    static constexpr int PASSES = PER == 8 ? kGateRows / 2 : kGateRows;
    static constexpr int ROWS_PER_WARP = RPP * PASSES;
};

template <int DV, int YT, int ZT>
__global__ void __launch_bounds__(32 * kGateWarps)
out_gate_kernel(const void* __restrict__ y, const void* __restrict__ z, const float* __restrict__ w, float eps,
                long long rows, void* __restrict__ out) {
    using S = GateShape<DV, YT, ZT>;
    constexpr int PER = S::PER, LPR = S::LPR, R = S::PASSES;
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPR, c0 = (lane % LPR) * PER;
    const long long r0 = ((long long)blockIdx.x * kGateWarps + (threadIdx.x >> 5)) * S::ROWS_PER_WARP + sub;
    if (r0 - sub >= rows) return;
    float wv[PER], yv[R][PER], zv[R][PER], ss[R];
#pragma unroll
    for (int u = 0; u < PER; ++u) wv[u] = 1.0f + w[c0 + u];
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const long long r = r0 + (long long)i * S::RPP;
        if (r < rows) {
            ldv<YT, PER>(y, (size_t)r * DV + c0, yv[i]);
            ldv<ZT, PER>(z, (size_t)r * DV + c0, zv[i]);
        } else {
#pragma unroll
            for (int u = 0; u < PER; ++u) yv[i][u] = zv[i][u] = 0.f;
        }
        ss[i] = 0.f;
#pragma unroll
        for (int u = 0; u < PER; ++u) ss[i] += yv[i][u] * yv[i][u];
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) {
#pragma unroll
        for (int i = 0; i < R; ++i) ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], o);
    }
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const float inv = rsqrtf(ss[i] / DV + eps);
#pragma unroll
        for (int u = 0; u < PER; ++u) yv[i][u] = __fdividef(yv[i][u] * inv * wv[u], 1.0f + __expf(-zv[i][u]));
    }
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const long long r = r0 + (long long)i * S::RPP;
        if (r < rows) stv<ZT, PER>(out, (size_t)r * DV + c0, yv[i]);
    }
}

}  // namespace gdn
