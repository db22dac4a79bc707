// decode.cuh -- one token per row against a resident fp32 state, eqs. (1)-(4) of
// "On the design of Qwen3.8-Next architecture", section 2.1.1 ("Gated Delta recurrence").
//
// Work per (row, head): one streaming pass over the dk x dv fp32 state.  The update is
// rewritten so that a single read and a single write of S suffice:
//   a = S^T k, b = S^T q                 (both from the same sweep over S)
//   e = v - alpha a                      (eq. 2 with S~ = alpha S, eq. 1)
//   S <- alpha S + beta k e^T            (eq. 3), written back in place
//   y = scale (alpha b + beta (k.q) e)   (eq. 4: S_t^T q expanded, no second pass)
// The kernel is HBM-bound (about 0.9 FLOP per byte): one CTA per (row, head).  Thread 0 brings
// the state block into shared memory with one bulk copy first; every thread then reads RPT rows
// x 4 columns of it twice (the two dot products, then the update) and streams the new state out
// with 128-bit stores.  With the state in shared memory rather than registers, three CTAs share
// an SM, so one CTA's reductions overlap the others' state traffic.
#pragma once
#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdn {

template <int DK, int DV>
struct DecodeShape {
    static constexpr int CPR = DV / 4;                   // float4 columns per state row
    static constexpr int RG0 = 256 / CPR;                // row groups at 256 threads
    static constexpr int RG = RG0 < DK ? RG0 : DK;       // row groups actually used
    static constexpr int THREADS = CPR * RG;
    static constexpr int RPT = DK / RG;                  // rows per thread
};

template <int DK, int DV>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::THREADS, 3)
decode_step_kernel(const void* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
                   const float* __restrict__ g, const float* __restrict__ beta, float* __restrict__ state,
                   const int32_t* __restrict__ slot, int num_slots, int H, float scale, int in_dt,
                   int y_dt, void* __restrict__ y, unsigned long long budget) {
    using Sh = DecodeShape<DK, DV>;
    const int bh = blockIdx.x;  // row * H + head
    const int b = bh / H, h = bh - b * H;
    const int tid = threadIdx.x;
    const int cq = tid % Sh::CPR;  // float4 column index
    const int rg = tid / Sh::CPR;  // row group

    __shared__ float s_k[DK], s_q[DK], s_v[DV], s_e[DV];
    __shared__ float4 s_red_a[Sh::RG][Sh::CPR], s_red_b[Sh::RG][Sh::CPR];
    __shared__ float s_kq;

    int s = slot ? slot[b] : b;
    if (s < 0 || s >= num_slots) {  // uniform across the block
        if (tid == 0) raise_error(kErrSlot);
        return;
    }
    // (bounds-checking build) the state block and the token row lie inside their tensors
    if (!in_bounds(((long long)s * H + h + 1) * DK * DV - 1, (long long)num_slots * H * DK * DV) ||
        !in_bounds(bh, (long long)gridDim.x))
        return;
    float* S = state + ((size_t)s * H + h) * DK * DV;

    // The state first: it is the only traffic that matters.  One bulk copy of the dk x dv block;
    // the barrier's initialisation is visible to the other threads after the __syncthreads
    // below, before any of them waits on it.
    extern __shared__ __align__(16) float s_st[];  // [DK][DV]
    __shared__ __align__(8) uint64_t s_bar;
    if (tid == 0) {
        tc::mbar_init(&s_bar, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(&s_bar, DK * DV * 4);
        tc::bulk_g2s(s_st, S, DK * DV * 4, &s_bar);
    }

    for (int i = tid; i < DK; i += Sh::THREADS) {
        s_k[i] = ld1(k, in_dt, (size_t)bh * DK + i);
        s_q[i] = ld1(q, in_dt, (size_t)bh * DK + i);
    }
    for (int j = tid; j < DV; j += Sh::THREADS) s_v[j] = ld1(v, in_dt, (size_t)bh * DV + j);
    const float alpha = expf(g[bh]);
    const float bt = beta[bh];
    __syncthreads();

    if (tid < 32) {
        float p = 0.f;
        for (int i = tid; i < DK; i += 32) p += s_k[i] * s_q[i];
        p = warp_sum(p);
        if (tid == 0) s_kq = p;
    }

    if (!tc::mbar_wait_bounded(&s_bar, 0, budget)) {  // flag it, and let the copy land
        if (tid == 0) raise_error(kErrTimeout);
        tc::mbar_wait_bounded(&s_bar, 0, 4000000000ull);
    }
    const float4* st = reinterpret_cast<const float4*>(s_st);  // row i, float4 column cq: st[i * CPR + cq]
    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
    for (int m = 0; m < Sh::RPT; ++m) {
        const int i = rg + m * Sh::RG;
        const float ki = s_k[i], qi = s_q[i];
        const float4 sv4 = st[i * Sh::CPR + cq];
        pa.x += sv4.x * ki; pa.y += sv4.y * ki; pa.z += sv4.z * ki; pa.w += sv4.w * ki;
        pb.x += sv4.x * qi; pb.y += sv4.y * qi; pb.z += sv4.z * qi; pb.w += sv4.w * qi;
    }
    s_red_a[rg][cq] = pa;
    s_red_b[rg][cq] = pb;
    __syncthreads();

    if (tid < DV) {  // column totals, e and y for column j = tid
        const int j = tid, c4 = j >> 2, l = j & 3;
        float a = 0.f, bb = 0.f;
#pragma unroll 8
        for (int r = 0; r < Sh::RG; ++r) {
            a += reinterpret_cast<const float*>(&s_red_a[r][c4])[l];
            bb += reinterpret_cast<const float*>(&s_red_b[r][c4])[l];
        }
        const float e = s_v[j] - alpha * a;
        s_e[j] = e;
        st1(y, y_dt, (size_t)bh * DV + j, scale * (alpha * bb + bt * s_kq * e));
    }
    __syncthreads();

    const float4 e4 = reinterpret_cast<const float4*>(s_e)[cq];
#pragma unroll
    for (int m = 0; m < Sh::RPT; ++m) {
        const int i = rg + m * Sh::RG;
        const float w = bt * s_k[i];
        const float4 sv4 = st[i * Sh::CPR + cq];
        float4 o;
        o.x = alpha * sv4.x + w * e4.x;
        o.y = alpha * sv4.y + w * e4.y;
        o.z = alpha * sv4.z + w * e4.z;
        o.w = alpha * sv4.w + w * e4.w;
        __stcs(reinterpret_cast<float4*>(S + (size_t)i * DV) + cq, o);
    }
}

}  // namespace gdn
