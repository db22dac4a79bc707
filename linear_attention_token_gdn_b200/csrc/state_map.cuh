// state_map.cuh -- a sequence segment's affine map on the state, the exchange unit of
// context-parallel prefill.
//
// Eqs. (1)-(3) of "On the design of Qwen3.8-Next architecture", section 2.1.1, combine into
// the closed form eq. (5): S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, which
// is affine in S_{t-1}.  Over a segment of tokens the composition stays affine:
//     S_end = M S_start + B,
// M (dk x dk) = the product of the per-token factors alpha_t (I - beta_t k_t k_t^T), i.e. the
// segment run from S = I with v = 0, and B (dk x dv) = the segment run from S = 0.  A rank that
// holds one segment of a sequence gets its initial state by applying the maps of the segments
// before it, in order, to the sequence's initial state.
//
// state_map_kernel: S_out = M S_in + B for each state row, fp32 on the CUDA cores (the maps are
// 64 KiB per head and applied once per segment: a few MFLOP per head, nothing to tile for).  One
// CTA per 16 x 16 output tile, dk staged through shared memory 16 columns at a time.
#pragma once
#include "common.cuh"

namespace gdn {

__global__ void __launch_bounds__(256) state_map_kernel(const float* __restrict__ M, const float* __restrict__ B,
                                                        const float* __restrict__ S_in, float* __restrict__ S_out,
                                                        int dk, int dv) {
    __shared__ float sm[16][17], ss[16][17];
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int tj_n = dv / 16, tiles = (dk / 16) * tj_n;
    const long long blk = blockIdx.x;
    const long long b = blk / tiles;
    const int t = (int)(blk - b * tiles), ti = t / tj_n, tj = t - ti * tj_n;
    const float* Mb = M + b * dk * dk;
    const float* Sb = S_in + b * dk * dv;
    float acc = 0.f;
    for (int k0 = 0; k0 < dk; k0 += 16) {
        sm[ty][tx] = Mb[(size_t)(16 * ti + ty) * dk + k0 + tx];
        ss[ty][tx] = Sb[(size_t)(k0 + ty) * dv + 16 * tj + tx];
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 16; ++k) acc = fmaf(sm[ty][k], ss[k][tx], acc);
        __syncthreads();
    }
    const size_t o = (size_t)b * dk * dv + (size_t)(16 * ti + ty) * dv + 16 * tj + tx;
    S_out[o] = acc + (B != nullptr ? B[o] : 0.f);
}

}  // namespace gdn
