// prep.cuh -- eqs. (6)-(10) of "On the design of Qwen3.8-Next architecture", section 2.1.1
// ("GDN parameterisation"): causal depthwise ShortConv -> SiLU (-> L2Norm for q, k) on the
// projection outputs, and the per-head beta / log-alpha gates.
//
// One CTA per (run of kPrepRun tokens, head), heads fastest across the grid.  One TMA copy per
// tensor brings the run's q, k, v input rows and the conv history before it into shared memory
// (about 50 KB in flight per CTA for bf16, so the SM keeps enough bytes moving to stream at HBM
// speed).  Two warps take each tensor, one per half of the run: a lane owns d/32 adjacent
// channels, keeps their taps and the last W-1 rows in registers and computes 8 independent
// tokens at a time (L2Norm is a warp reduction); warp 6 forms the gates.  HBM-bound: 3 x d inputs and outputs per (token, head).
#pragma once
#include "common.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace gdn {

constexpr int kPrepRun = 64;    // tokens per CTA
constexpr int kPrepBatch = 4;   // input rows loaded per batch

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

// `per` adjacent channels of one input row held in shared memory (input format IDT).
template <int PER, int IDT>
__device__ __forceinline__ void lds_row(const uint8_t* p, float (&x)[PER]) {
    if constexpr (IDT == kF32) {
        if constexpr (PER == 4) {
            const float4 v = *reinterpret_cast<const float4*>(p);
            x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
        } else {
#pragma unroll
            for (int u = 0; u < PER; ++u) x[u] = reinterpret_cast<const float*>(p)[u];
        }
    } else {
        constexpr bool BF = IDT == kBF16;
        if constexpr (PER == 4) {
            const uint2 v = *reinterpret_cast<const uint2*>(p);
            const float2 a = unpack2<BF>(v.x), b = unpack2<BF>(v.y);
            x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
        } else if constexpr (PER == 2) {
            const float2 a = unpack2<BF>(*reinterpret_cast<const uint32_t*>(p));
            x[0] = a.x; x[1] = a.y;
        } else {
            const uint16_t v = *reinterpret_cast<const uint16_t*>(p);
            x[0] = unpack2<BF>((uint32_t)v).x;
        }
    }
}

// The batches of one tensor over tokens [t0, t1).  CLEAN: the window [t0 - (TAPS - 1), t1) lies
// in one sequence, so no tap is masked and no token needs its sequence start.
template <int D, int TAPS, bool NORM, int IDT, bool CLEAN>
__device__ __forceinline__ void prep_batches(const uint8_t* __restrict__ row0, const float (&wp)[TAPS][D >= 32 ? D / 32 : 1],
                                             float (&xb)[TAPS - 1 + kPrepBatch][D >= 32 ? D / 32 : 1], void* __restrict__ out,
                                             int out_dt, float eps, int t0, int t1, int H, int h, int c0, bool active,
                                             SeqWalk& sw) {
    constexpr int PER = D >= 32 ? D / 32 : 1;
    constexpr int HIST = TAPS - 1;
    constexpr int B = kPrepBatch;
    constexpr int ESZ = IDT == kF32 ? 4 : 2;
#pragma unroll 1
    for (int tb = t0; tb < t1; tb += B) {
        const int rb = tb - t0 + HIST;  // tile row of token tb
#pragma unroll
        for (int k = 0; k < B; ++k) {
            if (active && tb + k < t1) lds_row<PER, IDT>(row0 + (rb + k) * D * ESZ, xb[HIST + k]);
            else {
#pragma unroll
                for (int u = 0; u < PER; ++u) xb[HIST + k][u] = 0.f;
            }
        }
        int lim[B];  // previous tokens of the same sequence (unused when CLEAN)
        if constexpr (!CLEAN) {
#pragma unroll
            for (int k = 0; k < B; ++k) lim[k] = tb + k < t1 ? tb + k - sw.start_of(tb + k) : -1;
        }
        float y[B][PER];
#pragma unroll
        for (int k = 0; k < B; ++k) {
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                float acc = 0.f;
                if (CLEAN || lim[k] >= HIST) {
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
        size_t e = ((size_t)tb * H + h) * D + c0;
        const size_t step = (size_t)H * D;
#pragma unroll
        for (int k = 0; k < B; ++k, e += step)
            if (active && tb + k < t1) st_row<PER>(out, out_dt, e, y[k]);
#pragma unroll
        for (int i = 0; i < HIST; ++i) {
#pragma unroll
            for (int u = 0; u < PER; ++u) xb[i][u] = xb[B + i][u];
        }
    }
}

// One tensor (q, k or v) of one head over tokens [t0, t1), at most kPrepRun / 2 of them:
// ShortConv -> SiLU (-> L2Norm), read from the CTA's tile, whose row r holds token
// tt - (TAPS - 1) + r (rows before a sequence start are masked, rows before token 0 or past N
// are zero-filled by the copy).  The tokens of a batch are computed independently, so their
// reductions interleave.
template <int D, int TAPS, bool NORM, int IDT>
__device__ __forceinline__ void prep_tensor(const uint8_t* __restrict__ tile, int tt, const float* __restrict__ w,
                                            int W, void* __restrict__ out, int out_dt, float eps, int t0, int t1,
                                            int H, int h, int lane, SeqWalk sw) {
    constexpr int PER = D >= 32 ? D / 32 : 1;
    constexpr int HIST = TAPS - 1;
    constexpr int B = kPrepBatch;
    constexpr int ESZ = IDT == kF32 ? 4 : 2;
    const bool active = D >= 32 || lane < D;
    const int c0 = (D >= 32 ? lane * PER : lane);
    const uint8_t* row0 = tile + (t0 - tt) * D * ESZ + c0 * ESZ;  // row of token t0 - HIST + r at row0 + r * D * ESZ
    float wp[TAPS][PER];  // wp[TAPS - W + j] = w[c][j]
#pragma unroll
    for (int i = 0; i < TAPS; ++i) {
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int j = i - (TAPS - W);
            wp[i][u] = (active && j >= 0) ? w[((size_t)h * D + c0 + u) * W + j] : 0.f;
        }
    }
    float xb[HIST + B][PER];  // [0, HIST): the rows before the batch; then the batch
#pragma unroll
    for (int i = 0; i < HIST; ++i) {
        if (active) lds_row<PER, IDT>(row0 + i * D * ESZ, xb[i]);
        else {
#pragma unroll
            for (int u = 0; u < PER; ++u) xb[i][u] = 0.f;
        }
    }
    if constexpr (TAPS <= 4) {  // (the wider conv has no registers for a second copy of the loop)
        const int s0 = sw.start_of(t0);  // t0's sequence is [s0, sw.nxt)
        if (t0 - s0 >= HIST && t1 <= sw.nxt) {
            prep_batches<D, TAPS, NORM, IDT, true>(row0, wp, xb, out, out_dt, eps, t0, t1, H, h, c0, active, sw);
            return;
        }
    }
    prep_batches<D, TAPS, NORM, IDT, false>(row0, wp, xb, out, out_dt, eps, t0, t1, H, h, c0, active, sw);
}

// TMA descriptors of the three projection outputs, [N, H, d] each; box = d x 1 x (run + taps - 1).
struct PrepMaps {
    CUtensorMap q, k, v;
};

// Bytes of one tensor's tile (rows padded to a 128-byte multiple per tile).
__host__ __device__ constexpr int prep_tile_bytes(int D, int taps, int esz) {
    return ((kPrepRun + taps - 1) * D * esz + 127) / 128 * 128;
}

constexpr int kPrepThreads = 224;  // 2 warps per tensor + 1 for the gates

template <int DK, int DV, int TAPS>
__global__ void __launch_bounds__(kPrepThreads, 4)
prep_kernel(const __grid_constant__ PrepMaps maps, const float* __restrict__ wq, const float* __restrict__ wk,
            const float* __restrict__ wv, int W, const void* __restrict__ beta_logit,
            const void* __restrict__ alpha_logit, const float* __restrict__ A_log,
            const float* __restrict__ alpha_bias, const int32_t* __restrict__ cu, int num_seqs, int N, int H,
            float eps, int in_dt, int out_dt, void* __restrict__ q, void* __restrict__ k, void* __restrict__ v,
            float* __restrict__ g_out, float* __restrict__ beta_out, unsigned long long budget) {
    constexpr int HIST = TAPS - 1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((128u - (tc::smem_u32(smem_raw) & 127u)) & 127u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // heads vary fastest across the grid, so CTAs resident together read whole token rows
    const int h = (int)(blockIdx.x % (unsigned)H);
    const int t0 = (int)(blockIdx.x / (unsigned)H) * kPrepRun;
    SeqWalk sw;
    sw.init(cu, num_seqs, N, t0);
    const int t1 = min(t0 + kPrepRun, sw.stop);  // tokens past the last sequence stay untouched
    if (warp == 6 && blockIdx.x == 0 && cu != nullptr) {
        // the walk only meets the sequences this CTA covers: one warp checks them all
        // (cu[0] >= 0, non-decreasing, cu[num_seqs] <= N) and flags a malformed array
        bool bad = false;
        for (int m = lane; m < num_seqs; m += 32) bad |= cu[m] < 0 || cu[m + 1] < cu[m] || cu[m + 1] > N;
        if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(kErrSeqlens);
    }
    if (t0 >= t1) return;  // uniform over the CTA
    const int esz = in_dt == kF32 ? 4 : 2;
    const int tqk = prep_tile_bytes(DK, TAPS, esz), tv = prep_tile_bytes(DV, TAPS, esz);
    uint8_t* tile_q = smem;
    uint8_t* tile_k = smem + tqk;
    uint8_t* tile_v = smem + 2 * tqk;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 2 * tqk + tv);
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(bar, (uint32_t)((kPrepRun + HIST) * (2 * DK + DV) * esz));
        tc::tma_load_3d(tile_q, &maps.q, 0, h, t0 - HIST, bar);
        tc::tma_load_3d(tile_k, &maps.k, 0, h, t0 - HIST, bar);
        tc::tma_load_3d(tile_v, &maps.v, 0, h, t0 - HIST, bar);
    }
    __syncthreads();
    if (warp == 6) {  // the gates need no tile
        const float ea = expf(A_log[h]), bias = alpha_bias[h];
        for (int t = t0 + lane; t < t1; t += 32) {
            const size_t th = (size_t)t * H + h;
            beta_out[th] = 1.0f / (1.0f + expf(-ld1(beta_logit, in_dt, th)));     // eq. (9)
            g_out[th] = -ea * softplusf_(ld1(alpha_logit, in_dt, th) + bias);      // eq. (10)
        }
    }
    if (!tc::mbar_wait_bounded(bar, 0, budget)) {  // flag, let the copies land, skip the work
        if (lane == 0) raise_error(kErrTimeout);
        tc::mbar_wait_bounded(bar, 0, 4000000000ull);
        return;
    }
    if (warp == 6) return;
    const int ten = warp >> 1;  // 0 q, 1 k, 2 v
    const uint8_t* tile = ten == 0 ? tile_q : ten == 1 ? tile_k : tile_v;
    const float* w = ten == 0 ? wq : ten == 1 ? wk : wv;
    void* out = ten == 0 ? q : ten == 1 ? k : v;
    const int ta = t0 + (warp & 1) * (kPrepRun / 2), tb = min(ta + kPrepRun / 2, t1);
    if (ta >= tb) return;
    SeqWalk swh = sw;  // walks on from the run's first token: no second search
    swh.start_of(ta);
    // eqs. (6), (7): q and k are normalised; eq. (8): v is not
#define GDN_PREP_TENSOR(IDT)                                                                                     \
    if (ten < 2) prep_tensor<DK, TAPS, true, IDT>(tile, t0, w, W, out, out_dt, eps, ta, tb, H, h, lane, swh);   \
    else prep_tensor<DV, TAPS, false, IDT>(tile, t0, w, W, out, out_dt, eps, ta, tb, H, h, lane, swh);
    if (in_dt == kBF16) {
        GDN_PREP_TENSOR(kBF16)
    } else if (in_dt == kF16) {
        GDN_PREP_TENSOR(kF16)
    } else {
        GDN_PREP_TENSOR(kF32)
    }
#undef GDN_PREP_TENSOR
}

}  // namespace gdn
