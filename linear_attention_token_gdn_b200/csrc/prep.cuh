// prep.cuh -- eqs. (6)-(10) of "On the design of Qwen3.8-Next architecture", section 2.1.1
// ("GDN parameterisation"): causal depthwise ShortConv -> SiLU (-> L2Norm for q, k) on the
// projection outputs, and the per-head beta / log-alpha gates.
//
// One CTA per (run of kPrepRun tokens, head), heads fastest across the grid, four warps: q, k, v and the gates.  A tensor's
// warp walks its run; each lane owns d/32 adjacent channels (one 8-byte load per row for
// 16-bit inputs), keeps their conv taps and the last W-1 input rows in registers, so every
// input row is read from memory once (plus the history rows of each run).  L2Norm is a
// warp reduction.  Rows are read and computed in batches of 8 independent tokens, which keeps
// loads and reductions in flight.  HBM-bound: 3 x d inputs and outputs per (token, head).
#pragma once
#include "common.cuh"

namespace gdn {

constexpr int kPrepRun = 64;    // tokens per CTA
constexpr int kPrepBatch = 8;   // input rows loaded per batch

// `per` adjacent channels of one row, starting at element i.
template <int PER>
__device__ __forceinline__ void ld_row(const void* p, int dt, size_t i, float (&x)[PER]) {
    if constexpr (PER == 4) {
        const float4 v = ld4(p, dt, i);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
#pragma unroll
        for (int u = 0; u < PER; ++u) x[u] = ld1(p, dt, i + u);
    }
}

template <int PER>
__device__ __forceinline__ void st_row(void* p, int dt, size_t i, const float (&x)[PER]) {
    if constexpr (PER == 4) {
        st4(p, dt, i, make_float4(x[0], x[1], x[2], x[3]));
    } else {
#pragma unroll
        for (int u = 0; u < PER; ++u) st1(p, dt, i + u, x[u]);
    }
}

// Sequence bookkeeping of a warp walking tokens upward: [cur, nxt) is the sequence holding
// the current token; tokens at or past `stop` (the end of the last sequence) are not touched.
struct SeqWalk {
    const int32_t* cu;
    int num_seqs, N, L, m, cur, nxt, stop;

    __device__ void init(const int32_t* cu_, int num_seqs_, int N_, int t) {
        cu = cu_;
        num_seqs = num_seqs_;
        N = N_;
        if (cu == nullptr) {
            L = N / num_seqs;
            stop = L * num_seqs;
            m = L > 0 ? t / L : 0;
            cur = m * L;
            nxt = cur + L;
            return;
        }
        L = 0;
        stop = min(max(cu[num_seqs], 0), N);
        int lo = 0, hi = num_seqs - 1;  // the last m with cu[m] <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (cu[mid] <= t) lo = mid;
            else hi = mid - 1;
        }
        m = lo;
        seq_bounds(cu, m, num_seqs, N, cur, nxt);
    }
    // Start of t's sequence (t non-decreasing across calls, t < stop).
    __device__ int start_of(int t) {
        while (t >= nxt && m + 1 < num_seqs) {
            ++m;
            if (cu == nullptr) {
                cur = m * L;
                nxt = cur + L;
            } else {
                seq_bounds(cu, m, num_seqs, N, cur, nxt);
            }
        }
        return cur;
    }
};

// One tensor (q, k or v) of one head over tokens [t0, t1): ShortConv -> SiLU (-> L2Norm).
// TAPS >= conv width; the taps are zero-padded in front.  The tokens of a batch are computed
// independently (their reductions interleave), so each warp keeps 8 rows of work in flight.
template <int D, int TAPS, bool NORM>
__device__ __forceinline__ void prep_tensor(const void* __restrict__ x, const float* __restrict__ w, int W,
                                            void* __restrict__ out, int in_dt, int out_dt, float eps, int t0,
                                            int t1, int H, int h, int lane, SeqWalk sw) {
    constexpr int PER = D >= 32 ? D / 32 : 1;
    constexpr int HIST = TAPS - 1;
    constexpr int B = kPrepBatch;
    const bool active = D >= 32 || lane < D;
    const int c0 = (D >= 32 ? lane * PER : lane);
    float wp[TAPS][PER];  // wp[TAPS - W + j] = w[c][j]
#pragma unroll
    for (int i = 0; i < TAPS; ++i) {
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int j = i - (TAPS - W);
            wp[i][u] = (active && j >= 0) ? w[((size_t)h * D + c0 + u) * W + j] : 0.f;
        }
    }
    // xb[0 .. HIST-1]: the rows before the batch; xb[HIST ..]: the batch
    float xb[HIST + B][PER];
#pragma unroll
    for (int i = 0; i < HIST; ++i) {
        const int s = t0 - HIST + i;
#pragma unroll
        for (int u = 0; u < PER; ++u) xb[i][u] = 0.f;
        if (active && s >= 0) ld_row<PER>(x, in_dt, ((size_t)s * H + h) * D + c0, xb[i]);
    }
    for (int tb = t0; tb < t1; tb += B) {
#pragma unroll
        for (int k = 0; k < B; ++k) {
#pragma unroll
            for (int u = 0; u < PER; ++u) xb[HIST + k][u] = 0.f;
            if (active && tb + k < t1) ld_row<PER>(x, in_dt, ((size_t)(tb + k) * H + h) * D + c0, xb[HIST + k]);
        }
        int lim[B];  // previous tokens of the same sequence (-1: past t1)
#pragma unroll
        for (int k = 0; k < B; ++k) lim[k] = tb + k < t1 ? tb + k - sw.start_of(tb + k) : -1;
        float y[B][PER];
#pragma unroll
        for (int k = 0; k < B; ++k) {
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                float acc = 0.f;
                if (lim[k] >= HIST) {
#pragma unroll
                    for (int i = 0; i < TAPS; ++i) acc += wp[i][u] * xb[k + i][u];
                } else {
#pragma unroll
                    for (int i = 0; i < TAPS; ++i)
                        if (HIST - i <= lim[k]) acc += wp[i][u] * xb[k + i][u];
                }
                y[k][u] = __fdividef(acc, 1.0f + __expf(-acc));  // SiLU
            }
        }
        if constexpr (NORM) {
            float ss[B];
#pragma unroll
            for (int k = 0; k < B; ++k) {
                ss[k] = 0.f;
#pragma unroll
                for (int u = 0; u < PER; ++u) ss[k] += active ? y[k][u] * y[k][u] : 0.f;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
                for (int k = 0; k < B; ++k) ss[k] += __shfl_xor_sync(0xffffffffu, ss[k], o);
            }
#pragma unroll
            for (int k = 0; k < B; ++k) {
                const float inv = rsqrtf(ss[k] + eps);
#pragma unroll
                for (int u = 0; u < PER; ++u) y[k][u] *= inv;
            }
        }
#pragma unroll
        for (int k = 0; k < B; ++k)
            if (active && tb + k < t1) st_row<PER>(out, out_dt, ((size_t)(tb + k) * H + h) * D + c0, y[k]);
#pragma unroll
        for (int i = 0; i < HIST; ++i) {
#pragma unroll
            for (int u = 0; u < PER; ++u) xb[i][u] = xb[B + i][u];
        }
    }
}

template <int DK, int DV, int TAPS>
__global__ void __launch_bounds__(128)
prep_kernel(const void* __restrict__ xq, const void* __restrict__ xk, const void* __restrict__ xv,
            const float* __restrict__ wq, const float* __restrict__ wk, const float* __restrict__ wv, int W,
            const void* __restrict__ beta_logit, const void* __restrict__ alpha_logit,
            const float* __restrict__ A_log, const float* __restrict__ alpha_bias,
            const int32_t* __restrict__ cu, int num_seqs, int N, int H, float eps, int in_dt, int out_dt,
            void* __restrict__ q, void* __restrict__ k, void* __restrict__ v, float* __restrict__ g_out,
            float* __restrict__ beta_out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // heads vary fastest across the grid, so CTAs resident together read whole token rows
    const int h = (int)(blockIdx.x % (unsigned)H);
    const int t0 = (int)(blockIdx.x / (unsigned)H) * kPrepRun;
    SeqWalk sw;
    sw.init(cu, num_seqs, N, t0);
    const int t1 = min(t0 + kPrepRun, sw.stop);  // tokens past the last sequence stay untouched
    if (t0 >= t1) return;
    if (warp == 0) {
        prep_tensor<DK, TAPS, true>(xq, wq, W, q, in_dt, out_dt, eps, t0, t1, H, h, lane, sw);   // eq. (6)
    } else if (warp == 1) {
        prep_tensor<DK, TAPS, true>(xk, wk, W, k, in_dt, out_dt, eps, t0, t1, H, h, lane, sw);   // eq. (7)
    } else if (warp == 2) {
        prep_tensor<DV, TAPS, false>(xv, wv, W, v, in_dt, out_dt, eps, t0, t1, H, h, lane, sw);  // eq. (8)
    } else {
        const float ea = expf(A_log[h]), bias = alpha_bias[h];
        for (int t = t0 + lane; t < t1; t += 32) {
            const size_t th = (size_t)t * H + h;
            beta_out[th] = 1.0f / (1.0f + expf(-ld1(beta_logit, in_dt, th)));     // eq. (9)
            g_out[th] = -ea * softplusf_(ld1(alpha_logit, in_dt, th) + bias);      // eq. (10)
        }
    }
}

}  // namespace gdn
