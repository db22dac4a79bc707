// out_gate.cuh -- eq. (11) of "On the design of Qwen3.8-Next architecture", section 2.1.1,
// without the output projection W_o: out = sigmoid(z) * y / sqrt(mean(y^2) + eps) * (1 + w),
// the zero-centred RMSNorm over dv per (token, head) followed by the sigmoid output gate.
// One warp per (token, head); HBM-bound elementwise work.
#pragma once
#include "common.cuh"

namespace gdn {

constexpr int kGateWarps = 8;

template <int DV>
__global__ void __launch_bounds__(32 * kGateWarps)
out_gate_kernel(const void* __restrict__ y, const void* __restrict__ z, const float* __restrict__ w,
                float eps, long long rows, int y_dt, int io_dt, void* __restrict__ out) {
    constexpr int PER = DV >= 32 ? DV / 32 : 1;
    const int lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * kGateWarps + (threadIdx.x >> 5);
    if (r >= rows) return;
    float yv[PER];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int c = lane + 32 * u;
        yv[u] = c < DV ? ld1(y, y_dt, (size_t)r * DV + c) : 0.f;
        ss += yv[u] * yv[u];
    }
    const float inv = rsqrtf(warp_sum(ss) / DV + eps);
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int c = lane + 32 * u;
        if (c < DV) {
            const float zz = ld1(z, io_dt, (size_t)r * DV + c);
            st1(out, io_dt, (size_t)r * DV + c, yv[u] * inv * (1.0f + w[c]) / (1.0f + expf(-zz)));
        }
    }
}

}  // namespace gdn
