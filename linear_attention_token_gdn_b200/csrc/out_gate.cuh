// out_gate.cuh -- eq. (11) of "On the design of Qwen3.8-Next architecture", section 2.1.1,
// without the output projection W_o: out = sigmoid(z) * y / sqrt(mean(y^2) + eps) * (1 + w),
// the zero-centred RMSNorm over dv per (token, head) followed by the sigmoid output gate.
// One warp per kGateRows (token, head) rows; each lane owns dv/32 adjacent channels (vector
// loads), every row's y and z are loaded before the reductions, which interleave.
// HBM-bound elementwise work.
#pragma once
#include "common.cuh"

namespace gdn {

constexpr int kGateWarps = 8;
constexpr int kGateRows = 4;  // rows per warp

template <int DV>
__global__ void __launch_bounds__(32 * kGateWarps)
out_gate_kernel(const void* __restrict__ y, const void* __restrict__ z, const float* __restrict__ w,
                float eps, long long rows, int y_dt, int io_dt, void* __restrict__ out) {
    constexpr int PER = DV >= 32 ? DV / 32 : 1;
    constexpr int R = kGateRows;
    const int lane = threadIdx.x & 31;
    const bool active = DV >= 32 || lane < DV;
    const int c0 = DV >= 32 ? lane * PER : lane;
    const long long r0 = ((long long)blockIdx.x * kGateWarps + (threadIdx.x >> 5)) * R;
    if (r0 >= rows) return;
    float wv[PER], yv[R][PER], zv[R][PER], ss[R];
#pragma unroll
    for (int u = 0; u < PER; ++u) wv[u] = active ? 1.0f + w[c0 + u] : 0.f;
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const bool ok = active && r0 + i < rows;
        const size_t e = (size_t)(r0 + i) * DV + c0;
#pragma unroll
        for (int u = 0; u < PER; ++u) yv[i][u] = zv[i][u] = 0.f;
        if (ok) {
            if constexpr (PER == 4) {
                const float4 a = ld4(y, y_dt, e), b = ld4(z, io_dt, e);
                yv[i][0] = a.x; yv[i][1] = a.y; yv[i][2] = a.z; yv[i][3] = a.w;
                zv[i][0] = b.x; zv[i][1] = b.y; zv[i][2] = b.z; zv[i][3] = b.w;
            } else {
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    yv[i][u] = ld1(y, y_dt, e + u);
                    zv[i][u] = ld1(z, io_dt, e + u);
                }
            }
        }
        ss[i] = 0.f;
#pragma unroll
        for (int u = 0; u < PER; ++u) ss[i] += yv[i][u] * yv[i][u];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
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
        if (active && r0 + i < rows) {
            const size_t e = (size_t)(r0 + i) * DV + c0;
            if constexpr (PER == 4) {
                st4(out, io_dt, e, make_float4(yv[i][0], yv[i][1], yv[i][2], yv[i][3]));
            } else {
#pragma unroll
                for (int u = 0; u < PER; ++u) st1(out, io_dt, e + u, yv[i][u]);
            }
        }
    }
}

}  // namespace gdn
