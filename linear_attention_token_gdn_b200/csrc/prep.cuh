// prep.cuh -- eqs. (6)-(10) of "On the design of Qwen3.8-Next architecture", section 2.1.1
// ("GDN parameterisation"): causal depthwise ShortConv -> SiLU (-> L2Norm for q, k) on the
// projection outputs, and the per-head beta / log-alpha gates.
//
// One warp per (token, head).  Each lane owns d/32 channels of q, k and v; the W-1 history
// rows of each channel are re-read from global memory (they are the previous tokens' rows,
// already in L1/L2), with zeros before the sequence start.  L2Norm is a warp reduction.
// HBM-bound elementwise work: 3 x d inputs and outputs per (token, head).
#pragma once
#include "common.cuh"

namespace gdn {

constexpr int kPrepWarps = 8;

template <int D>
__device__ __forceinline__ void conv_silu_row(const void* x, const float* __restrict__ w, int W,
                                              int in_dt, int t, int t_start, int H, int h, int lane,
                                              float (&out)[D / 32]) {
    constexpr int PER = D / 32;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int c = lane + 32 * u;
        const float* wc = w + ((size_t)h * D + c) * W;
        float acc = 0.f;
        for (int jj = 0; jj < W; ++jj) {
            const int s = t - (W - 1) + jj;
            if (s >= t_start) acc += wc[jj] * ld1(x, in_dt, ((size_t)s * H + h) * D + c);
        }
        out[u] = acc / (1.0f + expf(-acc));  // SiLU
    }
}

template <int DK, int DV>
__global__ void __launch_bounds__(32 * kPrepWarps)
prep_kernel(const void* __restrict__ xq, const void* __restrict__ xk, const void* __restrict__ xv,
            const float* __restrict__ wq, const float* __restrict__ wk, const float* __restrict__ wv, int W,
            const void* __restrict__ beta_logit, const void* __restrict__ alpha_logit,
            const float* __restrict__ A_log, const float* __restrict__ alpha_bias,
            const int32_t* __restrict__ cu, int num_seqs, int N, int H, float eps, int in_dt, int out_dt,
            void* __restrict__ q, void* __restrict__ k, void* __restrict__ v, float* __restrict__ g_out,
            float* __restrict__ beta_out) {
    const int lane = threadIdx.x & 31;
    const long long th = (long long)blockIdx.x * kPrepWarps + (threadIdx.x >> 5);  // token*H + head
    if (th >= (long long)N * H) return;
    const int t = (int)(th / H), h = (int)(th % H);
    const int t_start = seq_start_of(cu, num_seqs, N, t);
    if (t_start < 0) return;  // past the last sequence: untouched

    float xr[DK / 32];
    conv_silu_row<DK>(xq, wq, W, in_dt, t, t_start, H, h, lane, xr);  // eq. (6)
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < DK / 32; ++u) ss += xr[u] * xr[u];
    float inv = rsqrtf(warp_sum(ss) + eps);
#pragma unroll
    for (int u = 0; u < DK / 32; ++u) st1(q, out_dt, (size_t)th * DK + lane + 32 * u, xr[u] * inv);

    conv_silu_row<DK>(xk, wk, W, in_dt, t, t_start, H, h, lane, xr);  // eq. (7)
    ss = 0.f;
#pragma unroll
    for (int u = 0; u < DK / 32; ++u) ss += xr[u] * xr[u];
    inv = rsqrtf(warp_sum(ss) + eps);
#pragma unroll
    for (int u = 0; u < DK / 32; ++u) st1(k, out_dt, (size_t)th * DK + lane + 32 * u, xr[u] * inv);

    float vr[DV / 32];
    conv_silu_row<DV>(xv, wv, W, in_dt, t, t_start, H, h, lane, vr);  // eq. (8)
#pragma unroll
    for (int u = 0; u < DV / 32; ++u) st1(v, out_dt, (size_t)th * DV + lane + 32 * u, vr[u]);

    if (lane == 0) {
        beta_out[th] = 1.0f / (1.0f + expf(-ld1(beta_logit, in_dt, th)));                 // eq. (9)
        g_out[th] = -expf(A_log[h]) * softplusf_(ld1(alpha_logit, in_dt, th) + alpha_bias[h]);  // eq. (10)
    }
}

// Head sizes below 32 use one lane per channel and a partial-warp reduction.
template <int DK, int DV>
__global__ void __launch_bounds__(32 * kPrepWarps)
prep_small_kernel(const void* __restrict__ xq, const void* __restrict__ xk, const void* __restrict__ xv,
                  const float* __restrict__ wq, const float* __restrict__ wk, const float* __restrict__ wv,
                  int W, const void* __restrict__ beta_logit, const void* __restrict__ alpha_logit,
                  const float* __restrict__ A_log, const float* __restrict__ alpha_bias,
                  const int32_t* __restrict__ cu, int num_seqs, int N, int H, float eps, int in_dt,
                  int out_dt, void* __restrict__ q, void* __restrict__ k, void* __restrict__ v,
                  float* __restrict__ g_out, float* __restrict__ beta_out) {
    const int lane = threadIdx.x & 31;
    const long long th = (long long)blockIdx.x * kPrepWarps + (threadIdx.x >> 5);
    if (th >= (long long)N * H) return;
    const int t = (int)(th / H), h = (int)(th % H);
    const int t_start = seq_start_of(cu, num_seqs, N, t);
    if (t_start < 0) return;

    auto conv = [&](const void* x, const float* w, int d, int c) {
        float acc = 0.f;
        if (c < d) {
            const float* wc = w + ((size_t)h * d + c) * W;
            for (int jj = 0; jj < W; ++jj) {
                const int s = t - (W - 1) + jj;
                if (s >= t_start) acc += wc[jj] * ld1(x, in_dt, ((size_t)s * H + h) * d + c);
            }
        }
        return acc / (1.0f + expf(-acc));
    };
    float xq_ = conv(xq, wq, DK, lane);
    float inv = rsqrtf(warp_sum(lane < DK ? xq_ * xq_ : 0.f) + eps);
    if (lane < DK) st1(q, out_dt, (size_t)th * DK + lane, xq_ * inv);
    float xk_ = conv(xk, wk, DK, lane);
    inv = rsqrtf(warp_sum(lane < DK ? xk_ * xk_ : 0.f) + eps);
    if (lane < DK) st1(k, out_dt, (size_t)th * DK + lane, xk_ * inv);
    float xv_ = conv(xv, wv, DV, lane);
    if (lane < DV) st1(v, out_dt, (size_t)th * DV + lane, xv_);
    if (lane == 0) {
        beta_out[th] = 1.0f / (1.0f + expf(-ld1(beta_logit, in_dt, th)));
        g_out[th] = -expf(A_log[h]) * softplusf_(ld1(alpha_logit, in_dt, th) + alpha_bias[h]);
    }
}

}  // namespace gdn
