// bwd.cuh -- reverse-mode derivative of eqs. (1)-(4) of "On the design of Qwen3.8-Next
// architecture", section 2.1.1, token-sequential in fp32 on the CUDA cores.
//
// For a loss L with dL/dy_t = dy_t and dL/dS_T = dS_T, each token step
//     S~ = alpha S,  e = v - S~^T k,  S_t = S~ + beta k e^T,  y = scale S_t^T q
// (S = S_{t-1}, alpha = exp(g)) is walked backwards with D = dL/dS_t:
//     D += scale q dy^T,  dq = scale S_t dy,  de = beta D^T k,  dbeta = k^T D e,
//     dk = beta D e - S~ de,  dv = de,  D~ = D - k de^T,  dg = alpha <D~, S>,  D <- alpha D~
// and dS0 is D after the first token.  A forward pass (recurrent_fwd_kernel with checkpoints)
// stores the state before every kBwdBlk-th token; this kernel walks each sequence's blocks from
// the last, recomputes the block's states into shared memory and walks them backwards.
//
// One CTA per (sequence, head, slab of state columns): thread (column jl, row phase r) keeps rows
// r, r + RS, ... of its column of D and of the block's states.  de, dv and the column's share of dbeta and dg need only the column; dq and dk sum over
// every column, so each CTA adds its slab's part through a shared-memory transpose and atomicAdd
// into fp32 outputs the caller has zeroed (the slabs' order of addition is not fixed).
#pragma once
#include "common.cuh"
#include "recurrent.cuh"

namespace gdn {

template <int DK, int DV>
struct BwdShape {
    // the forward kernel's column slabs; 16 rows per thread (8 for dk = 16)
    static constexpr int SLAB = RecShape<DK, DV>::SLAB;
    static constexpr int RS = DK >= 32 ? DK / 16 : 2;             // threads per column (2, 4 or 8)
    static constexpr int RPT = DK / RS;                           // rows per thread
    static constexpr int THREADS = SLAB * RS;
    // row stride of the transposes: a warp writes RS rows x 32/RS columns, and with a stride of
    // 4 (mod 32) words those land in 32 distinct banks; the readers rotate their start column by
    // lane so that a warp's 32 rows also read 32 distinct banks
    static constexpr int PAD = SLAB + 4;
    // tokens walked between two reductions: each has its own transposes and column sums, so that
    // one pair of barriers serves them all
    static constexpr int NP = 2;
    // shared memory: the block's states, the block's token inputs, NP x (two transposes, column sums)
    static constexpr int ST_FLOATS = kBwdBlk * DK * SLAB;
    static constexpr int TOK_FLOATS = kBwdBlk * (2 * DK + 2 * SLAB + 2);
    static constexpr int RED_ONE = 2 * DK * PAD + 2 * SLAB;
    static constexpr int RED_FLOATS = NP * RED_ONE;
    static constexpr int BYTES = 4 * (ST_FLOATS + TOK_FLOATS + RED_FLOATS);
};

template <int DK, int DV>
__global__ void __launch_bounds__(BwdShape<DK, DV>::THREADS)
recurrent_bwd_kernel(const void* __restrict__ q, const void* __restrict__ k, const void* __restrict__ v,
                     const float* __restrict__ g, const float* __restrict__ beta, const int32_t* __restrict__ cu,
                     int num_seqs, int N, int H, float scale, int in_dt, const void* __restrict__ dy, int dy_dt,
                     const float* __restrict__ dS_T, const float* __restrict__ ckpt, float* __restrict__ dq,
                     float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dg,
                     float* __restrict__ dbeta, float* __restrict__ dS0) {
    using Sh = BwdShape<DK, DV>;
    constexpr int NSLAB = DV / Sh::SLAB, SLAB = Sh::SLAB, RPT = Sh::RPT, RS = Sh::RS, NT = Sh::THREADS;
    constexpr int B = kBwdBlk;
    extern __shared__ float smem_f[];
    float* st = smem_f;                                  // [B][RPT][THREADS]: S before token tb + i, thread-major
    float* sk = st + Sh::ST_FLOATS;                      // [B][DK]
    float* sq = sk + B * DK;                             // [B][DK]
    float* sv = sq + B * DK;                             // [B][SLAB]
    float* sdy = sv + B * SLAB;                          // [B][SLAB]
    float* sa = sdy + B * SLAB;                          // [B] alpha
    float* sb = sa + B;                                  // [B] beta
    // NP slots of: [DK][PAD] the slab's terms of dq, [DK][PAD] of dk, [SLAB] the columns' terms of
    // dbeta, [SLAB] of dg / alpha
    float* p_q0 = sb + B;
    __shared__ int s_bbase;

    const int slab = blockIdx.x % NSLAB;
    const int h = (blockIdx.x / NSLAB) % H;
    const int n = blockIdx.x / (NSLAB * H);
    const int tid = threadIdx.x, jl = tid / RS, r = tid % RS, j = slab * SLAB + jl;
    int t0, t1;
    seq_bounds(cu, n, num_seqs, N, t0, t1);
    if (tid == 0) s_bbase = blocks_before(cu, num_seqs, N, n);

    const size_t sbase = ((size_t)n * H + h) * DK * DV;
    float D[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) D[m] = dS_T ? dS_T[sbase + (size_t)(r + m * RS) * DV + j] : 0.f;
    int nb = (t1 - t0 + B - 1) / B;
    __syncthreads();  // s_bbase
    if (s_bbase + (long long)nb > bwd_block_bound(N, num_seqs)) {  // malformed cu_seqlens: no block past the workspace
        if (tid == 0) raise_error(kErrSeqlens);
        nb = (int)max(0LL, bwd_block_bound(N, num_seqs) - s_bbase);
    }

    for (int b = nb - 1; b >= 0; --b) {
        const int tb = t0 + b * B, nt = min(B, t1 - tb);
        // (bounds-checking build) the block's tokens and checkpoint lie inside their tensors;
        // uniform over the CTA
        if (!in_bounds(tb, N) || !in_bounds(tb + nt - 1, N) || !in_bounds(s_bbase + b, bwd_block_bound(N, num_seqs)))
            break;
        __syncthreads();  // the previous block's token inputs are no longer read (and s_bbase is set)
        for (int idx = tid; idx < nt * DK; idx += NT) {
            const int tt = idx / DK, i = idx % DK;
            const size_t off = ((size_t)(tb + tt) * H + h) * DK + i;
            sk[tt * DK + i] = ld1(k, in_dt, off);
            sq[tt * DK + i] = ld1(q, in_dt, off);
        }
        for (int idx = tid; idx < nt * SLAB; idx += NT) {
            const int tt = idx / SLAB, jj = idx % SLAB;
            const size_t off = ((size_t)(tb + tt) * H + h) * DV + slab * SLAB + jj;
            sv[tt * SLAB + jj] = ld1(v, in_dt, off);
            sdy[tt * SLAB + jj] = ld1(dy, dy_dt, off);
        }
        for (int tt = tid; tt < nt; tt += NT) {
            sa[tt] = expf(g[(size_t)(tb + tt) * H + h]);
            sb[tt] = beta[(size_t)(tb + tt) * H + h];
        }
        __syncthreads();
        // the block's states, recomputed from its checkpoint; each thread keeps the entries it owns
        {
            const float* cp = ckpt + ((size_t)(s_bbase + b) * H + h) * DK * DV;
            float S[RPT];
#pragma unroll
            for (int m = 0; m < RPT; ++m) S[m] = cp[(size_t)(r + m * RS) * DV + j];
            for (int i = 0; i < nt; ++i) {
                float a = 0.f;
#pragma unroll
                for (int m = 0; m < RPT; ++m) {
                    st[(i * RPT + m) * NT + tid] = S[m];
                    a += S[m] * sk[i * DK + r + m * RS];
                }
#pragma unroll
                for (int o = 1; o < RS; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                const float e = sv[i * SLAB + jl] - sa[i] * a;
#pragma unroll
                for (int m = 0; m < RPT; ++m) S[m] = sa[i] * S[m] + sb[i] * sk[i * DK + r + m * RS] * e;
            }
        }
        // tokens i, i - 1, ... (NP of them) are walked back to back, each into its own transposes;
        // one barrier, then their column sums, then a barrier before the next group overwrites them
        for (int i0 = nt - 1; i0 >= 0; i0 -= Sh::NP) {
            const int np = min(Sh::NP, i0 + 1);
#pragma unroll
            for (int sl = 0; sl < Sh::NP; ++sl) {
                if (sl >= np) break;  // uniform
                const int i = i0 - sl, t = tb + i;
                float* p_q = p_q0 + sl * Sh::RED_ONE;
                float* p_k = p_q + DK * Sh::PAD;
                float* c_b = p_k + DK * Sh::PAD;
                float* c_g = c_b + SLAB;
                const float alpha = sa[i], bt = sb[i], dyj = sdy[i * SLAB + jl];
                float kk[RPT], qq[RPT];  // this thread's rows of k_t and q_t
#pragma unroll
                for (int m = 0; m < RPT; ++m) {
                    kk[m] = sk[i * DK + r + m * RS];
                    qq[m] = sq[i * DK + r + m * RS];
                }
                float Sp[RPT], a = 0.f;
#pragma unroll
                for (int m = 0; m < RPT; ++m) {
                    Sp[m] = st[(i * RPT + m) * NT + tid];
                    a += Sp[m] * kk[m];
                }
#pragma unroll
                for (int o = 1; o < RS; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                const float e = sv[i * SLAB + jl] - alpha * a;
                float kd = 0.f;
#pragma unroll
                for (int m = 0; m < RPT; ++m) {
                    const int row = r + m * RS;
                    const float St = alpha * Sp[m] + bt * kk[m] * e;      // S_t
                    D[m] += scale * qq[m] * dyj;                            // readout
                    p_q[row * Sh::PAD + jl] = scale * St * dyj;             // dq = scale S_t dy
                    kd += kk[m] * D[m];
                }
#pragma unroll
                for (int o = 1; o < RS; o <<= 1) kd += __shfl_xor_sync(0xffffffffu, kd, o);
                const float de = bt * kd;                                   // de = beta D^T k
                float da = 0.f;
#pragma unroll
                for (int m = 0; m < RPT; ++m) {
                    const int row = r + m * RS;
                    p_k[row * Sh::PAD + jl] = bt * D[m] * e - alpha * Sp[m] * de;  // dk = beta D e - S~ de
                    D[m] -= kk[m] * de;                                     // D~
                    da += D[m] * Sp[m];
                    D[m] *= alpha;                                          // dL/dS_{t-1}
                }
#pragma unroll
                for (int o = 1; o < RS; o <<= 1) da += __shfl_xor_sync(0xffffffffu, da, o);
                if (r == 0) {
                    dv[((size_t)t * H + h) * DV + j] = de;
                    c_b[jl] = kd * e;                                       // dbeta = k^T D e
                    c_g[jl] = da;
                }
            }
            __syncthreads();
            // the slab's column terms: a row of dq or dk of one token per thread (four partial
            // sums), and dbeta, dg of each token by one warp
            for (int e = tid; e < np * 2 * DK; e += NT) {
                const int sl = e / (2 * DK), re = e - sl * 2 * DK;
                const int row = re < DK ? re : re - DK, t = tb + i0 - sl;
                const float* pr = p_q0 + sl * Sh::RED_ONE + (re < DK ? 0 : DK * Sh::PAD) + row * Sh::PAD;
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < SLAB; ++c) s4[c & 3] += pr[(c + tid) & (SLAB - 1)];
                atomicAdd((re < DK ? dq : dk) + ((size_t)t * H + h) * DK + row, (s4[0] + s4[1]) + (s4[2] + s4[3]));
            }
            for (int sl = tid >> 5; sl < np; sl += NT / 32) {  // (warp-uniform; NT is a multiple of 32)
                const int l = tid & 31, t = tb + i0 - sl;
                const float* c_b = p_q0 + sl * Sh::RED_ONE + 2 * DK * Sh::PAD;
                const float* c_g = c_b + SLAB;
                float s1 = l < SLAB ? c_b[l] : 0.f, s2 = l < SLAB ? c_g[l] : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
                    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
                }
                if (l == 0) {
                    atomicAdd(dbeta + (size_t)t * H + h, s1);
                    atomicAdd(dg + (size_t)t * H + h, sa[i0 - sl] * s2);
                }
            }
            __syncthreads();  // the transposes are read before the next group writes them
        }
    }
#pragma unroll
    for (int m = 0; m < RPT; ++m) dS0[sbase + (size_t)(r + m * RS) * DV + j] = D[m];
}

}  // namespace gdn
