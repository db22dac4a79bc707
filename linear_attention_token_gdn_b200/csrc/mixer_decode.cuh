// mixer_decode.cuh -- one token per row through the whole GDN mixer of "On the design of
// Qwen3.8-Next architecture", section 2.1.1, in one kernel:
//   eqs. (6)-(10)  causal ShortConv over the row's conv history + the token's projection
//                  outputs, SiLU, L2Norm for q and k; beta = sigmoid, g = log alpha
//   eqs. (1)-(4)   the gated delta rule against the resident fp32 state, in place
//   eq.  (11)      out = sigmoid(z) y / sqrt(mean(y^2) + eps) (1 + w), without W_o
// The conv history of each slot (the W-1 previous raw inputs, oldest first) is shifted in
// place, the current input appended.  Nothing between the steps goes to memory: q, k, v stay
// fp32 in shared memory.
//
// One CTA per (row, head).  Thread 0 brings the slot's whole state block into shared memory with
// one bulk copy before the prep arithmetic starts, so the prep work hides under it; the updated
// state is written back with 128-bit streaming stores.  Holding the state in shared memory rather
// than registers lets three CTAs share an SM, so that one CTA's prep and reductions overlap the
// others' state traffic.  HBM-bound: dk x dv x 8 bytes of state per (row, head), plus
// 2 (W-1) (2 dk + dv) bytes of conv history and the token's inputs and output.
#pragma once
#include "common.cuh"
#include "decode.cuh"
#include "tc_ptx.cuh"

namespace gdn {

struct MixerDecodeArgs {
    const void *x_q, *x_k, *x_v;
    const float *w_q, *w_k, *w_v;
    int W;
    const void *beta_logit, *alpha_logit;
    const float *A_log, *alpha_bias;
    const void* z;
    const float* norm_w;
    float l2_eps, rms_eps;
    void* conv_state;
    float* state;
    const int32_t* slot;
    int num_slots, H;
    float scale;
    int in_dt, out_dt;
    void* out;
    unsigned long long budget;  // clock cycles a wait may take before it is reported
};

// TAPS: the largest conv width the instantiation takes (4 or 8), so that the window lives in
// registers with static indices.
template <int DK, int DV, int TAPS>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::THREADS, TAPS == 4 ? 3 : 2)
    mixer_decode_kernel(const MixerDecodeArgs a) {
    using Sh = DecodeShape<DK, DV>;
    constexpr int NT = Sh::THREADS, CH = 2 * DK + DV;  // channels of one head's conv input
    const int bh = blockIdx.x;                         // row * H + head
    const int H = a.H, b = bh / H, h = bh - b * H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cq = tid % Sh::CPR, rg = tid / Sh::CPR;

    __shared__ float s_x[CH];          // q (dk), k (dk), v (dv) after conv + SiLU (+ L2Norm)
    __shared__ float s_e[DV], s_y[DV];
    __shared__ float4 s_red_a[Sh::RG][Sh::CPR], s_red_b[Sh::RG][Sh::CPR];
    __shared__ float s_sc[4];          // 1/|q|, 1/|k|, k.q, 1/rms(y)
    __shared__ float s_gate[2];        // alpha, beta

    const int s = a.slot ? a.slot[b] : b;
    if (s < 0 || s >= a.num_slots) {  // uniform across the block
        if (tid == 0) raise_error(kErrSlot);
        return;
    }
    // (bounds-checking build) the slot's state block lies inside the state tensor
    if (!in_bounds(((long long)s * H + h + 1) * DK * DV - 1, (long long)a.num_slots * H * DK * DV)) return;
    float* S = a.state + ((size_t)s * H + h) * DK * DV;

    // the state first: it is the traffic that matters.  One bulk copy of the dk x dv block; the
    // barrier's initialisation is visible to the other threads after the first __syncthreads below,
    // before any of them waits on it.
    extern __shared__ __align__(16) float s_st[];  // [DK][DV]
    __shared__ __align__(8) uint64_t s_bar;
    if (tid == 0) {
        tc::mbar_init(&s_bar, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(&s_bar, DK * DV * 4);
        tc::bulk_g2s(s_st, S, DK * DV * 4, &s_bar);
    }

    // ---- eqs. (6)-(8): ShortConv over [history, current] then SiLU, one channel per thread; the
    //      history is shifted in place (entry j <- entry j + 1, the current input last).  Every
    //      global load of this phase is issued before any arithmetic or store, so their latencies
    //      overlap each other and the state loads. ----------------------------------------------
    constexpr int CPT = (CH + NT - 1) / NT;     // channels per thread
    constexpr int HMAX = TAPS - 1;              // history entries at most
    const int W = a.W, HW = W - 1;
    const size_t hist_stride = (size_t)H * CH;  // elements between history entries of a slot
    const size_t hist0 = (size_t)s * HW * hist_stride + (size_t)h * CH;
    // (bounds-checking build) the slot's conv history lies inside its tensor; uniform over the CTA
    if (HW > 0 && !in_bounds((long long)hist0 + (long long)(HW - 1) * hist_stride + CH - 1,
                             (long long)a.num_slots * HW * hist_stride))
        return;
    float xw[CPT][HMAX], taps[CPT][HMAX];       // history oldest first, and its taps
    float xcur[CPT], tcur[CPT];                 // the current input and tap W-1
    float bl = 0.f, al = 0.f, Ah = 0.f, bh_ = 0.f;
    if (tid == 0) {
        bl = ld1(a.beta_logit, a.in_dt, bh);
        al = ld1(a.alpha_logit, a.in_dt, bh);
        Ah = a.A_log[h];
        bh_ = a.alpha_bias[h];
    }
#pragma unroll
    for (int u = 0; u < CPT; ++u) {
        const int c = tid + u * NT;
        if (c < CH) {
            const bool isq = c < DK, isk = !isq && c < 2 * DK;
            const int i = isq ? c : (isk ? c - DK : c - 2 * DK);
            const int d = isq || isk ? DK : DV;
            const void* xp = isq ? a.x_q : (isk ? a.x_k : a.x_v);
            const float* wp = (isq ? a.w_q : (isk ? a.w_k : a.w_v)) + ((size_t)h * d + i) * W;
#pragma unroll
            for (int j = 0; j < HMAX; ++j) {
                if (j < HW) {
                    taps[u][j] = wp[j];
                    xw[u][j] = ld1(a.conv_state, a.in_dt, hist0 + (size_t)j * hist_stride + c);
                }
            }
            tcur[u] = wp[W - 1];
            xcur[u] = ld1(xp, a.in_dt, (size_t)bh * d + i);
        }
    }
#pragma unroll
    for (int u = 0; u < CPT; ++u) {
        const int c = tid + u * NT;
        if (c < CH) {
            float acc = tcur[u] * xcur[u];  // tap W-1 meets the current token
#pragma unroll
            for (int j = 0; j < HMAX; ++j)
                if (j < HW) acc += taps[u][j] * xw[u][j];
            s_x[c] = acc / (1.f + __expf(-acc));  // SiLU
#pragma unroll
            for (int j = 0; j < HMAX; ++j) {  // entry j takes entry j + 1; the last the current input
                if (j < HW) {
                    float nx = xcur[u];
#pragma unroll
                    for (int jj = 0; jj < HMAX; ++jj)
                        if (jj == j + 1 && jj < HW) nx = xw[u][jj];
                    st1(a.conv_state, a.in_dt, hist0 + (size_t)j * hist_stride + c, nx);
                }
            }
        }
    }
    if (tid == 0) {  // eqs. (9)-(10)
        s_gate[1] = sigmoidf_(bl);
        s_gate[0] = expf(-expf(Ah) * softplusf_(al + bh_));
    }
    __syncthreads();
    // L2Norm of q (warp 0) and k (warp 1), and k.q (warp 2) once both are normalised
    if (warp < 2) {
        const float* x = s_x + warp * DK;
        float p = 0.f;
        for (int i = lane; i < DK; i += 32) p += x[i] * x[i];
        p = warp_sum(p);
        if (lane == 0) s_sc[warp] = rsqrtf(p + a.l2_eps);
    }
    __syncthreads();
    for (int i = tid; i < 2 * DK; i += NT) s_x[i] *= s_sc[i < DK ? 0 : 1];
    __syncthreads();
    if (warp == 0) {
        float p = 0.f;
        for (int i = lane; i < DK; i += 32) p += s_x[i] * s_x[DK + i];
        p = warp_sum(p);
        if (lane == 0) s_sc[2] = p;
    }
    const float* sq = s_x;
    const float* sk = s_x + DK;
    const float* sv = s_x + 2 * DK;
    const float alpha = s_gate[0], bt = s_gate[1];

    // ---- eqs. (1)-(4): a = S^T k and b = S^T q from one sweep, e = v - alpha a,
    //      S <- alpha S + beta k e^T, y = scale (alpha b + beta (k.q) e) ----------------------------
    if (!tc::mbar_wait_bounded(&s_bar, 0, a.budget)) {  // flag it, and let the copy land
        if (tid == 0) raise_error(kErrTimeout);
        tc::mbar_wait_bounded(&s_bar, 0, 4000000000ull);
    }
    const float4* st = reinterpret_cast<const float4*>(s_st);  // row i, float4 column cq: st[i * CPR + cq]
    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
    for (int m = 0; m < Sh::RPT; ++m) {
        const int i = rg + m * Sh::RG;
        const float ki = sk[i], qi = sq[i];
        const float4 sv4 = st[i * Sh::CPR + cq];
        pa.x += sv4.x * ki; pa.y += sv4.y * ki; pa.z += sv4.z * ki; pa.w += sv4.w * ki;
        pb.x += sv4.x * qi; pb.y += sv4.y * qi; pb.z += sv4.z * qi; pb.w += sv4.w * qi;
    }
    s_red_a[rg][cq] = pa;
    s_red_b[rg][cq] = pb;
    __syncthreads();
    if (tid < DV) {
        const int j = tid, c4 = j >> 2, l = j & 3;
        float av = 0.f, bv = 0.f;
#pragma unroll 8
        for (int r = 0; r < Sh::RG; ++r) {
            av += reinterpret_cast<const float*>(&s_red_a[r][c4])[l];
            bv += reinterpret_cast<const float*>(&s_red_b[r][c4])[l];
        }
        const float e = sv[j] - alpha * av;
        s_e[j] = e;
        s_y[j] = a.scale * (alpha * bv + bt * s_sc[2] * e);
    }
    __syncthreads();
    const float4 e4 = reinterpret_cast<const float4*>(s_e)[cq];
#pragma unroll
    for (int m = 0; m < Sh::RPT; ++m) {
        const int i = rg + m * Sh::RG;
        const float wk = bt * sk[i];
        const float4 sv4 = st[i * Sh::CPR + cq];
        float4 o;
        o.x = alpha * sv4.x + wk * e4.x;
        o.y = alpha * sv4.y + wk * e4.y;
        o.z = alpha * sv4.z + wk * e4.z;
        o.w = alpha * sv4.w + wk * e4.w;
        __stcs(reinterpret_cast<float4*>(S + (size_t)i * DV) + cq, o);
    }

    // ---- eq. (11): out = sigmoid(z) y / sqrt(mean(y^2) + eps) (1 + w) -------------------------
    if (warp == 0) {
        float p = 0.f;
        for (int j = lane; j < DV; j += 32) p += s_y[j] * s_y[j];
        p = warp_sum(p);
        if (lane == 0) s_sc[3] = rsqrtf(p / DV + a.rms_eps);
    }
    __syncthreads();
    if (tid < DV) {
        const int j = tid;
        const float zj = ld1(a.z, a.in_dt, (size_t)bh * DV + j);
        st1(a.out, a.out_dt, (size_t)bh * DV + j, sigmoidf_(zj) * s_y[j] * s_sc[3] * (1.f + a.norm_w[j]));
    }
}

}  // namespace gdn
