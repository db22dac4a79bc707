// recurrent.cuh -- token-sequential prefill on CUDA cores, eqs. (1)-(4) of
// "On the design of Qwen3.8-Next architecture", section 2.1.1, in fp32.
//
// The state columns evolve independently (e_j depends only on column j of S), so one CTA
// owns a slab of SLAB state columns of one (sequence, head) and walks the sequence token
// by token.  Thread (j, r) keeps rows r, r+RS, r+2RS, ... of column j in registers; the
// RS threads of a column are adjacent lanes and combine their partial dot products with
// shuffles.  Token inputs are staged in shared memory TILE tokens at a time.
// This path serves any supported head size and fp32 inputs; the tensor-core chunked
// path covers dk = dv = 128 with 16-bit inputs.
#pragma once
#include "common.cuh"

namespace gdn {

constexpr int kBwdBlk = 8;  // tokens between the backward's checkpoints

// Upper bound of the checkpoint blocks of all sequences (the workspace's size); it holds for every
// valid cu_seqlens.
__host__ __device__ inline long long bwd_block_bound(int N, int num_seqs) {
    return (N + kBwdBlk - 1) / kBwdBlk + num_seqs;
}

// Checkpoint blocks of sequences 0 .. n-1 (one thread; CTAs of these kernels may be narrower
// than a warp).
__device__ __forceinline__ int blocks_before(const int32_t* cu, int num_seqs, int N, int n) {
    int s = 0;
    for (int m = 0; m < n; ++m) {
        int a, b;
        seq_bounds(cu, m, num_seqs, N, a, b);
        s += (b - a + kBwdBlk - 1) / kBwdBlk;
    }
    return s;
}

template <int DK, int DV>
struct RecShape {
    static constexpr int SLAB = DV < 32 ? DV : 32;         // state columns per CTA
    static constexpr int RPT = DK < 16 ? DK : 16;          // rows per thread
    static constexpr int RS = DK / RPT;                    // threads per column (1, 2, 4 or 8)
    static constexpr int THREADS = SLAB * RS;
    static constexpr int TILE = 32;                        // tokens staged per refill
};

template <int DK, int DV>
__global__ void __launch_bounds__(RecShape<DK, DV>::THREADS)
recurrent_fwd_kernel(const void* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
                     const float* __restrict__ g, const float* __restrict__ beta,
                     const float* __restrict__ S0, const int32_t* __restrict__ cu, int num_seqs, int N,
                     int H, float scale, int in_dt, int y_dt, void* __restrict__ y, float* __restrict__ S_T,
                     float* __restrict__ ckpt = nullptr) {
    using Sh = RecShape<DK, DV>;
    constexpr int NSLAB = DV / Sh::SLAB;
    const int slab = blockIdx.x % NSLAB;
    const int h = (blockIdx.x / NSLAB) % H;
    const int n = blockIdx.x / (NSLAB * H);
    const int tid = threadIdx.x;
    const int jl = tid / Sh::RS;             // local column
    const int r = tid % Sh::RS;              // row phase
    const int j = slab * Sh::SLAB + jl;      // global column

    __shared__ float s_k[Sh::TILE][DK], s_q[Sh::TILE][DK], s_v[Sh::TILE][Sh::SLAB];
    __shared__ float s_a[Sh::TILE], s_b[Sh::TILE];

    int t0, t1;
    seq_bounds(cu, n, num_seqs, N, t0, t1);
    // ckpt (the backward's checkpoints): the state before every kBwdBlk-th token of the sequence,
    // [block of all sequences in order][H][DK][DV]; y may then be NULL
    __shared__ int s_bbase;
    if (ckpt != nullptr) {
        if (tid == 0) s_bbase = blocks_before(cu, num_seqs, N, n);
        __syncthreads();
    }

    float S[Sh::RPT];
    const size_t sbase = ((size_t)n * H + h) * DK * DV;
#pragma unroll
    for (int m = 0; m < Sh::RPT; ++m) S[m] = S0 ? S0[sbase + (size_t)(r + m * Sh::RS) * DV + j] : 0.f;

    for (int tb = t0; tb < t1; tb += Sh::TILE) {
        const int nt = min(Sh::TILE, t1 - tb);
        // (bounds-checking build) the tile's tokens lie inside [0, N); uniform over the CTA
        if (!in_bounds(tb, N) || !in_bounds(tb + nt - 1, N)) break;
        __syncthreads();
        for (int idx = tid; idx < nt * DK; idx += Sh::THREADS) {
            const int tt = idx / DK, i = idx % DK;
            const size_t off = ((size_t)(tb + tt) * H + h) * DK + i;
            s_k[tt][i] = ld1(k, in_dt, off);
            s_q[tt][i] = ld1(q, in_dt, off);
        }
        for (int idx = tid; idx < nt * Sh::SLAB; idx += Sh::THREADS) {
            const int tt = idx / Sh::SLAB, jj = idx % Sh::SLAB;
            s_v[tt][jj] = ld1(v, in_dt, ((size_t)(tb + tt) * H + h) * DV + slab * Sh::SLAB + jj);
        }
        for (int tt = tid; tt < nt; tt += Sh::THREADS) {
            s_a[tt] = expf(g[(size_t)(tb + tt) * H + h]);
            s_b[tt] = beta[(size_t)(tb + tt) * H + h];
        }
        __syncthreads();

        for (int tt = 0; tt < nt; ++tt) {
            const long long blk = (long long)s_bbase + (tb + tt - t0) / kBwdBlk;
            // (malformed cu_seqlens, already flagged, could describe more blocks than the workspace)
            if (ckpt != nullptr && (tb + tt - t0) % kBwdBlk == 0 && blk < bwd_block_bound(N, num_seqs)) {
                float* cp = ckpt + ((size_t)blk * H + h) * DK * DV;
#pragma unroll
                for (int m = 0; m < Sh::RPT; ++m) cp[(size_t)(r + m * Sh::RS) * DV + j] = S[m];
            }
            const float alpha = s_a[tt], bt = s_b[tt];
            float a = 0.f;
#pragma unroll
            for (int m = 0; m < Sh::RPT; ++m) a += S[m] * s_k[tt][r + m * Sh::RS];
#pragma unroll
            for (int o = 1; o < Sh::RS; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            const float e = s_v[tt][jl] - alpha * a;          // eq. (2) with eq. (1)
            float yb = 0.f;
#pragma unroll
            for (int m = 0; m < Sh::RPT; ++m) {
                const int i = r + m * Sh::RS;
                S[m] = alpha * S[m] + bt * s_k[tt][i] * e;   // eq. (3)
                yb += S[m] * s_q[tt][i];                     // eq. (4), updated state
            }
#pragma unroll
            for (int o = 1; o < Sh::RS; o <<= 1) yb += __shfl_xor_sync(0xffffffffu, yb, o);
            if (r == 0 && y != nullptr) st1(y, y_dt, ((size_t)(tb + tt) * H + h) * DV + j, scale * yb);
        }
    }
    if (S_T) {
#pragma unroll
        for (int m = 0; m < Sh::RPT; ++m) S_T[sbase + (size_t)(r + m * Sh::RS) * DV + j] = S[m];
    }
}

}  // namespace gdn
