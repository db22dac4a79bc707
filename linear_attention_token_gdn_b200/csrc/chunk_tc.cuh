// chunk_tc.cuh -- chunkwise-parallel GDN prefill on the sm_100a tensor cores.
//
// The recurrence is eqs. (1)-(4) of "On the design of Qwen3.8-Next architecture", section
// 2.1.1.  Unrolling eqs. (1)-(3) over a chunk of C = 64 tokens that starts from state S
// (the closed form eq. (5) applied C times), with gamma_r the inclusive prefix sum of
// g = log alpha inside the chunk and Gamma_r = exp(gamma_r), gives
//     A[r,s] = beta_r exp(gamma_r - gamma_s) k_r.k_s   (s < r),   T = (I + A)^-1
//     W  = T diag(beta Gamma) K,      U~ = T diag(beta) V,      U = U~ - W S
//     M[r,s] = exp(gamma_r - gamma_s) q_r.k_s           (s <= r)
//     Y  = diag(Gamma) Q S + M U,     S' = Gamma_C S + K^T diag(Gamma_C / Gamma) U
// Every decay factor is exp(<= 0) and is applied elementwise to fp32 products, never
// factored as Gamma_r / Gamma_s.  For s in an earlier 16-row block than r the factor is
// split at the end e of s's block, exp(gamma_r - gamma_e) * exp(gamma_e - gamma_s), both
// factors <= 1, so a row needs 4 + 16 exponentials instead of 64.
//
// Two kernels:
//   chunk_ut_kernel     one CTA per (chunk, head), fully parallel, four CTAs per SM.
//                       [K;Q] K^T on tcgen05 (the 16-bit inputs used directly as
//                       operands), the decay masks, and the unit-lower-triangular inverse
//                       T in fp32 on the CUDA cores.  Writes a 24 KB record per
//                       (chunk, head): T_w = T diag(beta Gamma), T_u = T diag(beta) and M,
//                       already in the 128B-swizzled operand layout.
//   chunk_chain_kernel  one CTA per (sequence, head, 32-column dv slab), sequential over
//                       the chunks.  A producer warpgroup brings each chunk's K, Q and V
//                       tiles in with TMA, straight into operand slots, and computes
//                       W = T_w K and [0; U~] = [0; T_u] V on the tensor cores; a chain
//                       warpgroup carries the fp32 state (one row per thread) through two
//                       dependent tensor-core round trips per chunk:
//                           [0; U~] + [Q; -W] S -> Q S and U = U~ - W S in one accumulator
//                           K^T U'              -> S' = Gamma_C S + K^T U'
//                       with U' = diag(Gamma_C / Gamma) U, while M U, for
//                       Y = Gamma (Q S) + M U, is issued once the next chunk's [Q; -W] S
//                       has completed, when the MMA front end is otherwise idle.
//                       Q/W/M slots are double-buffered, K/V stages triple-buffered, all
//                       handed over with mbarriers; full chunks of y leave through swizzled
//                       TMA stores.  It is launched as a programmatic dependent of
//                       chunk_ut_kernel.  The gated variant applies eq. (11)'s output gate
//                       in the y epilogue, the four slab CTAs of a (sequence, head) forming
//                       one cluster that exchanges row sums of squares.
// Operands are 16-bit with fp32 accumulation in TMEM.  Each tcgen05.mma instruction costs
// the SM's MMA front end about as much below N = 128 as at N = 128, so products are shaped
// to use few instructions.  q and k enter exactly as stored (bf16 or fp16), so their partners
// (T_w, W, S, U') take the same format; U' enters as a rounded high half plus its remainder,
// side by side in one N = 64 operand, because its rounding would show in the state.  Products
// between values we compute -- T_u V (V converted to fp16 in place) and M U -- run in fp16
// (11 significant bits).
// Operand tiles use the 128B / 64B swizzled canonical layouts, so one tile serves as K-major
// or MN-major operand.  Every wait is bounded (ChunkArgs::budget clock cycles); a wait that
// runs out sets the device error word, lets in-flight MMAs and copies drain, and the CTA
// returns after freeing TMEM.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace gdn {

struct ChunkArgs {
    const void *q, *k, *v;
    const float *g, *beta, *S0;
    const int32_t* cu;
    int num_seqs, N, H, chunk;
    float scale;
    int in_dt, y_dt;
    void* y;
    float* S_T;
    void* workspace;
    unsigned long long budget;
    // fused output gate (gdn_chunk_fwd_gated): out = sigmoid(z) y / rms(y) (1 + norm_w), and y
    // is not written.  Unused (out == nullptr) by gdn_chunk_fwd.
    const void* z;
    const float* norm_w;
    float eps;
    int z_dt;
    void* out;
};

// TMA descriptors of the chain kernel: [N, H, 128] views of k, q (64-column halves, 128B
// swizzle), v and z (NS-column slab, 64B swizzle) and y -- or out, when the gate is fused --
// (NS-column slab stores, swizzled to the row width).
struct ChainMaps {
    CUtensorMap k, q, v, y, z;
};

constexpr int kChunk = 64;
// Record of one (chunk, head), written by chunk_ut_kernel: three [64 rows x 128 B] operand tiles
// in the 128B-swizzled K-major layout.
constexpr int kRecTw = 0;          // T_w = T diag(beta Gamma), 16-bit in the input's format (meets K)
constexpr int kRecTu = 8192;       // T_u = T diag(beta), fp16 (meets V converted to fp16)
constexpr int kRecM = 16384;       // M, fp16 (meets U, another computed operand)
constexpr int kRecBytes = 24576;

// Upper bound of the number of 64-token chunks over all sequences (the records the workspace
// holds); it holds for every valid cu_seqlens.
__host__ __device__ inline long long chunk_count_bound(int N, int num_seqs, bool varlen) {
    if (!varlen) {
        const long long L = N / num_seqs;
        return (long long)num_seqs * ((L + kChunk - 1) / kChunk);
    }
    return (N + kChunk - 1) / kChunk + num_seqs;
}

inline size_t chunk_tc_workspace_bytes(int N, int num_seqs, int H, int, int, int chunk) {
    if (chunk != kChunk || N <= 0 || num_seqs <= 0 || H <= 0) return 0;
    // the bound for packed sequences also covers equal lengths
    return (size_t)chunk_count_bound(N, num_seqs, true) * H * kRecBytes;
}

// Chunks of sequence m (warp-uniform).
__device__ __forceinline__ int seq_chunks(const int32_t* cu, int m, int num_seqs, int N) {
    int a, b;
    seq_bounds(cu, m, num_seqs, N, a, b);
    return (b - a + kChunk - 1) / kChunk;
}

// Virtual chunk v -> (sequence n, chunk j of n).  Warp-collective; false if v is past the end.
__device__ bool locate_chunk(const int32_t* cu, int num_seqs, int N, int v, int& n, int& j) {
    const int lane = threadIdx.x & 31;
    int base = 0;
    for (int m0 = 0; m0 < num_seqs; m0 += 32) {
        const int m = m0 + lane;
        const int cnt = m < num_seqs ? seq_chunks(cu, m, num_seqs, N) : 0;
        int inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += t;
        }
        const int total = __shfl_sync(0xffffffffu, inc, 31);
        if (v < base + total) {
            const unsigned hit = __ballot_sync(0xffffffffu, base + inc > v);
            const int l = __ffs(hit) - 1;
            n = m0 + l;
            j = v - (base + __shfl_sync(0xffffffffu, inc, l) - __shfl_sync(0xffffffffu, cnt, l));
            return true;
        }
        base += total;
    }
    return false;
}

// Number of chunks of sequences 0 .. n-1 (warp-collective).
__device__ int chunks_before(const int32_t* cu, int num_seqs, int N, int n) {
    const int lane = threadIdx.x & 31;
    int s = 0;
    for (int m0 = 0; m0 < n; m0 += 32) {
        const int m = m0 + lane;
        s += m < n ? seq_chunks(cu, m, num_seqs, N) : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// The dynamic shared-memory base rounded up to 1024 bytes (the swizzle atom of the operand
// tiles).  Offsetting the __shared__ array itself keeps the pointer in the shared address
// space, so every access through it compiles to a shared-memory load or store.
__device__ __forceinline__ uint8_t* align_smem_1024(uint8_t* raw) {
    return raw + ((1024u - (tc::smem_u32(raw) & 1023u)) & 1023u);
}

// Descriptor of the same operand advanced by byte_off (the start-address field holds
// address >> 4 in its low 14 bits; operands stay below 256 KB, so no carry leaves the field).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t byte_off) { return d + (byte_off >> 4); }

__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void sts4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

template <bool BF>
__device__ __forceinline__ uint4 pack8(const float* x) {
    return make_uint4(pack2<BF>(x[0], x[1]), pack2<BF>(x[2], x[3]), pack2<BF>(x[4], x[5]), pack2<BF>(x[6], x[7]));
}

// x = hi + lo + O(2^-16 |x|) for bf16 (2^-22 for fp16): hi = round(x), lo = round(x - hi).
template <bool BF>
__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        h[i] = pack2<BF>(x[2 * i], x[2 * i + 1]);
        const float2 f = unpack2<BF>(h[i]);
        l[i] = pack2<BF>(x[2 * i] - f.x, x[2 * i + 1] - f.y);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

template <bool BF>
__host__ __device__ constexpr uint32_t idesc16(int M, int N, bool a_mn, bool b_mn) {
    return BF ? tc::idesc_bf16(M, N, a_mn, b_mn) : tc::idesc_f16(M, N, a_mn, b_mn);
}

__device__ __forceinline__ void st16(uint8_t* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

// =====================================================================================
// chunk_ut_kernel: per (chunk, head) -- masks and the UT transform
// =====================================================================================

struct UtCfg {
    static constexpr int LD = 68;                           // fp32 row stride of A and T
    static constexpr int OFF_KQ = 0;                        // [K;Q] as stored: 2 x [128 x 128 B]
    static constexpr int OFF_A = 0;                         // fp32 A [64][LD], over [K;Q] once read
    static constexpr int OFF_Z = OFF_A + 64 * LD * 4;       // fp32 Z [3][16][20], likewise
    static constexpr int OFF_T = 32768;                     // fp32 T [64][LD]
    static constexpr int OFF_VEC = OFF_T + 64 * LD * 4;     // gamma, Gamma, beta, colf: 4 x 64
    static constexpr int OFF_META = OFF_VEC + 1024;
    static constexpr int OFF_BAR = OFF_META + 32;
    static constexpr int BYTES = OFF_BAR + 32 + 1024;
    static_assert(OFF_Z + 3 * 16 * 20 * 4 <= OFF_T, "A and Z fit in the [K;Q] tiles");
    static constexpr uint32_t TMEM_COLS = 64;
};

template <bool BF>
__global__ void __launch_bounds__(128, 4) chunk_ut_kernel(const __grid_constant__ ChunkArgs a,
                                                          const __grid_constant__ ChainMaps maps) {
    using Cf = UtCfg;
    constexpr int LD = Cf::LD;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    const uint32_t sbase = tc::smem_u32(smem);
    float* fA = reinterpret_cast<float*>(smem + Cf::OFF_A);
    float* fT = reinterpret_cast<float*>(smem + Cf::OFF_T);
    float* fZ = reinterpret_cast<float*>(smem + Cf::OFF_Z);
    float* vb = reinterpret_cast<float*>(smem + Cf::OFF_VEC);  // gamma[0:64] Gamma[64:128] beta[128:192] colf[192:256]
    int* meta = reinterpret_cast<int*>(smem + Cf::OFF_META);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cf::OFF_BAR);       // MMA done
    uint64_t* bar_ld = bar + 1;                                            // K, Q tiles landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::OFF_BAR + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // heads vary fastest across the grid, so CTAs resident together read whole token rows
    const int H = a.H, v = (int)(blockIdx.x / (unsigned)H), h = (int)(blockIdx.x % (unsigned)H);
    tc::launch_dependents();  // the chain kernel may start its prologue once every CTA is resident
    if (warp == 0) {
        int n = 0, j = 0;
        const bool found = locate_chunk(a.cu, a.num_seqs, a.N, v, n, j);
        if (lane == 0) {
            meta[0] = found;
            meta[1] = n;
            meta[2] = j;
        }
    }
    __syncthreads();
    if (!meta[0]) return;
    int t_begin, t_end;
    seq_bounds(a.cu, meta[1], a.num_seqs, a.N, t_begin, t_end);
    const int t0 = t_begin + meta[2] * kChunk, L = min(kChunk, t_end - t0);
    uint8_t* rec = reinterpret_cast<uint8_t*>(a.workspace) + ((size_t)v * H + h) * kRecBytes;

    // ---- K (rows 0-63) and Q (rows 64-127) as they are stored (bf16 or fp16), by TMA into the
    //      128B-swizzled operand layout.  Rows past the sequence end hold other tokens; they
    //      only meet beta = 0 or the strictly-upper mask, so nothing needs clearing. ----------------
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(bar_ld, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(bar_ld, 4 * 8192);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tc::tma_load_3d(smem + Cf::OFF_KQ + hf * 16384, &maps.k, 64 * hf, h, t0, bar_ld);
            tc::tma_load_3d(smem + Cf::OFF_KQ + hf * 16384 + 8192, &maps.q, 64 * hf, h, t0, bar_ld);
        }
    }
    if (tid < 64) {
        float gv = tid < L ? a.g[(size_t)(t0 + tid) * H + h] : 0.f;
        vb[128 + tid] = tid < L ? a.beta[(size_t)(t0 + tid) * H + h] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, gv, o);
            if (lane >= o) gv += y;
        }
        vb[tid] = gv;
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, Cf::TMEM_COLS);
    __syncthreads();
    if (tid >= 32 && tid < 64) vb[tid] += vb[31];
    __syncthreads();
    if (tid < 64) {
        vb[64 + tid] = __expf(vb[tid]);
        vb[192 + tid] = __expf(vb[tid | 15] - vb[tid]);  // exp(gamma_e - gamma_s), e = end of s's block
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool landed = __syncthreads_and(tc::mbar_wait_bounded(bar_ld, 0, a.budget)) != 0;
    if (!landed) {
        if (tid == 0) raise_error(kErrTimeout);
        tc::mbar_wait_bounded(bar_ld, 0, 4000000000ull);
    }

    // ---- [K;Q] K^T ---------------------------------------------------------------------------
    if (tid == 0 && landed) {
        constexpr uint32_t id = idesc16<BF>(128, 64, false, false);
        const uint64_t d0 = tc::smem_desc(sbase + Cf::OFF_KQ, 16, 1024, tc::kSw128);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t d = desc_add(d0, (kk >> 2) * 16384 + (kk & 3) * 32);
            tc::mma_f16(tmem, d, d, id, kk > 0);
        }
        tc::mma_commit(bar);
    }
    bool done = false;
    if (landed) {  // uniform
        done = __syncthreads_and(tc::mbar_wait_bounded(bar, 0, a.budget)) != 0;
        if (!done) {
            if (tid == 0) raise_error(kErrTimeout);
            tc::mbar_wait_bounded(bar, 0, 4000000000ull);
        }
    }
    tc::tc_fence_after();

    if (landed && done) {
        // ---- masks: A (fp32, over the consumed [K;Q] tiles) for the solve; M (fp16) straight
        //      into the record ---------------------------------------------------------------------
        {
            float x[64];
            const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
            tc::tmem_ld32(trow, x);
            tc::tmem_ld32(trow + 32, x + 32);
            const int r = tid & 63, R = r >> 4, rl = r & 15;
            const float gr = vb[r];
            const bool isA = tid < 64;
            float rowf[4], dg[16];
#pragma unroll
            for (int S = 0; S < 4; ++S) rowf[S] = S < R ? __expf(gr - vb[16 * S + 15]) : 0.f;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) dg[jj] = (isA ? jj < rl : jj <= rl) ? __expf(gr - vb[16 * R + jj]) : 0.f;
            const float sc = isA ? vb[128 + r] : 1.f;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                float m[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = 8 * cc + e, S = s >> 4;
                    const float f = S < R ? rowf[S] * vb[192 + s] : (S == R ? dg[s & 15] : 0.f);
                    m[e] = sc * f * x[s];
                }
                if (isA) {
                    sts4(fA + r * LD + 8 * cc, make_float4(m[0], m[1], m[2], m[3]));
                    sts4(fA + r * LD + 8 * cc + 4, make_float4(m[4], m[5], m[6], m[7]));
                } else {
                    st16(rec + kRecM + tc::swz_off(r, cc, 128), pack8<false>(m));
                }
            }
        }
        __syncthreads();

        // ---- T = (I + A)^-1: 16x16 diagonal blocks by forward substitution (lane = column) -----
        if (lane < 16) {
            const int b0 = warp * 16, jc = lane;
            float xs[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float arow[16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 t = lds4(fA + (b0 + r) * LD + b0 + 4 * q4);
                    arow[4 * q4] = t.x; arow[4 * q4 + 1] = t.y; arow[4 * q4 + 2] = t.z; arow[4 * q4 + 3] = t.w;
                }
                float acc = (r == jc) ? 1.f : 0.f;
#pragma unroll
                for (int s = 0; s < r; ++s) acc -= arow[s] * xs[s];
                xs[r] = acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) fT[(b0 + r) * LD + b0 + jc] = xs[r];
        }
        __syncthreads();
        // off-diagonal blocks, d = i - j = 1, 2, 3:  T_ij = -T_ii sum_{m=j}^{i-1} A_im T_mj
        // work item = (block, row rr, 4-column group cg)
        for (int d = 1; d < 4; ++d) {
            const int items = (4 - d) * 64;
            for (int o = tid; o < items; o += 128) {
                const int blk = o >> 6, i = d + blk, jb = i - d, rr = (o >> 2) & 15, cg = o & 3;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int m = jb; m < i; ++m) {
#pragma unroll
                    for (int s4 = 0; s4 < 4; ++s4) {
                        const float4 av = lds4(fA + (16 * i + rr) * LD + 16 * m + 4 * s4);
                        const float a4[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float4 t = lds4(fT + (16 * m + 4 * s4 + e) * LD + 16 * jb + 4 * cg);
                            acc.x += a4[e] * t.x; acc.y += a4[e] * t.y; acc.z += a4[e] * t.z; acc.w += a4[e] * t.w;
                        }
                    }
                }
                sts4(fZ + (blk * 16 + rr) * 20 + 4 * cg, acc);
            }
            __syncthreads();
            for (int o = tid; o < items; o += 128) {
                const int blk = o >> 6, i = d + blk, jb = i - d, rr = (o >> 2) & 15, cg = o & 3;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    const float4 tv = lds4(fT + (16 * i + rr) * LD + 16 * i + 4 * s4);
                    const float t4[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s = 4 * s4 + e;
                        const float tt = s <= rr ? t4[e] : 0.f;
                        const float4 z = lds4(fZ + (blk * 16 + s) * 20 + 4 * cg);
                        acc.x -= tt * z.x; acc.y -= tt * z.y; acc.z -= tt * z.z; acc.w -= tt * z.w;
                    }
                }
                sts4(fT + (16 * i + rr) * LD + 16 * jb + 4 * cg, acc);
            }
            __syncthreads();
        }
        // ---- T_w = T diag(beta Gamma) (input's format), T_u = T diag(beta) (fp16) -> record ------
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int idx = tid + 128 * u, which = idx >> 9, r = (idx >> 3) & 63, cc = idx & 7;
            const float4 t0v = lds4(fT + r * LD + 8 * cc), t1v = lds4(fT + r * LD + 8 * cc + 4);
            const float4 b0v = lds4(vb + 128 + 8 * cc), b1v = lds4(vb + 128 + 8 * cc + 4);
            float t8[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
            float s8[8] = {b0v.x, b0v.y, b0v.z, b0v.w, b1v.x, b1v.y, b1v.z, b1v.w};
            if (which == 0) {
                const float4 g0v = lds4(vb + 64 + 8 * cc), g1v = lds4(vb + 64 + 8 * cc + 4);
                s8[0] *= g0v.x; s8[1] *= g0v.y; s8[2] *= g0v.z; s8[3] *= g0v.w;
                s8[4] *= g1v.x; s8[5] *= g1v.y; s8[6] *= g1v.z; s8[7] *= g1v.w;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) t8[e] = (8 * cc + e <= r) ? t8[e] * s8[e] : 0.f;
            if (which == 0) st16(rec + kRecTw + tc::swz_off(r, cc, 128), pack8<BF>(t8));
            else st16(rec + kRecTu + tc::swz_off(r, cc, 128), pack8<false>(t8));
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, Cf::TMEM_COLS);
    }
}

// =====================================================================================
// chunk_chain_kernel: per (sequence, head, dv slab) -- the sequential pass over chunks
// =====================================================================================

template <int NS>
struct ChainCfg {
    static constexpr int ROWB = NS * 2;                        // bytes per row of a 16-bit slab tile
    static constexpr int UROWB = 2 * ROWB;                     // [hi | lo] rows of U': 128 B
    static constexpr uint32_t SWZ = NS == 32 ? tc::kSw64 : tc::kSw128;
    static constexpr int QW_HALF = 128 * 128;                  // one 64-column half of [Q;W]
    static constexpr int K_HALF = 64 * 128;                    // one 64-column half of K
    static constexpr int OFF_QW = 0;                           // [2 slots] [Q;W]: 2 halves x [128 x 128 B]
    static constexpr int OFF_M = OFF_QW + 2 * 2 * QW_HALF;     // [2 slots] M fp16: [64 x 128 B]
    static constexpr int OFF_KS = OFF_M + 2 * 8192;            // [3 stages] K: 2 halves x [64 x 128 B]
    static constexpr int OFF_TT = OFF_KS + 3 * 2 * K_HALF;     // [T_w; T_w; 0; T_u]: [256 x 128 B]
    static constexpr int OFF_VS = OFF_TT + 32768;              // [3 stages] V slab [64 x ROWB]
    static constexpr int OFF_SS = OFF_VS + 3 * 64 * ROWB;      // S [128 x ROWB]
    static constexpr int OFF_SU = OFF_SS + 128 * ROWB;         // [2 slots] U fp16: [64 x ROWB]
    static constexpr int OFF_SU2 = OFF_SU + 2 * 64 * ROWB;     // [U' hi | U' lo]: [64 x UROWB]
    static constexpr int OFF_YS = OFF_SU2 + 64 * UROWB;        // y rows for the TMA store [64 x NS x 4 B]
    static constexpr int OFF_ZS = OFF_YS + 64 * NS * 4;        // [2 slots] z slab [64 x ROWB] (gated)
    static constexpr int OFF_GZ = OFF_ZS + 2 * 64 * ROWB;      // sigmoid(z) (1 + w) rows, fp32 [64 x NS] (gated)
    static constexpr int OFF_VEC = OFF_GZ + 64 * NS * 4;       // [2 slots] gamma, Gamma, f: 3 x 64 floats
    static constexpr int OFF_META = OFF_VEC + 2 * 1024;        // [2 slots] {c0, L}
    static constexpr int OFF_RS = OFF_META + 64;               // [2] [4 slabs] [64 rows] y^2 sums (gated)
    static constexpr int OFF_NW = OFF_RS + 2 * 4 * 64 * 4;     // 1 + norm_w of this slab (gated)
    static constexpr int OFF_BAR = OFF_NW + NS * 4;
    static constexpr int NBARS = 22;
    static constexpr int BYTES = OFF_BAR + 256 + 1024;
    static constexpr uint32_t KV_TX = 2 * K_HALF + 64 * ROWB;  // K and the V slab of one chunk
    static constexpr uint32_t Q_TX = 2 * 8192;                 // Q of one chunk
    static constexpr uint32_t M_TX = 8192;                     // M of one chunk
    static constexpr uint32_t Z_TX = 64 * ROWB;                // z slab of one chunk (gated)
    // TMEM columns
    static constexpr uint32_t COL_U = 0;                       // [2 slots] x NS: [0; U~] + [Q; -W] S over dk 0-63
    static constexpr uint32_t COL_W = 2 * NS;                  // 128: W (both lane halves)
    static constexpr uint32_t COL_1B = COL_W + 128;            // NS: [Q; -W] S over dk 64-127
    static constexpr uint32_t COL_MU = COL_1B + NS;            // NS: M U (lanes 0-63)
    static constexpr uint32_t COL_DS = COL_MU + NS;            // 2 NS: [K^T U' hi | K^T U' lo]
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(COL_DS + 2 * NS <= TMEM_COLS, "TMEM budget");
    static_assert(NS == 32, "[hi | lo] operand rows are one 128-byte swizzle atom");
    static_assert(NBARS * 8 <= 192, "barrier area");
    static_assert(BYTES <= 232448, "shared memory budget");
    static_assert(OFF_M % 1024 == 0 && OFF_KS % 1024 == 0 && OFF_TT % 1024 == 0 && OFF_YS % 1024 == 0 &&
                      OFF_VS % 1024 == 0 && OFF_SS % 1024 == 0 && OFF_SU % 1024 == 0 && OFF_SU2 % 1024 == 0 && OFF_ZS % 1024 == 0 &&
                      OFF_GZ % 1024 == 0,
                  "swizzle atoms");
};

// Synchronisation of one chunk c in slot b = c & 1 (stage c % 3 for K and V):
//   producer -> chain   full[b]      W(c) in [Q;W] slot b, U~(c) in TMEM, gates and bounds of c
//                       q[b], m[b]   Q(c), M(c) landed (TMA / bulk copy bytes)
//   chain -> producer   ds_done[b]   the state MMA of c completed: [Q;W] slot b, U~ columns b and
//                                    K stage c % 3 are free (everything else of c was read before)
//                       m_empty[b]   M U of c completed: M slot b and U slot b are free
// The chain issues M U of chunk c once chunk c + 1's [Q;W] S has completed (the MMA front end is
// idle while warps 2-3 form U) and forms y of c meanwhile.
template <int NS, bool BF, bool GATED>
__global__ void __launch_bounds__(256, 1) chunk_chain_kernel(const __grid_constant__ ChunkArgs a,
                                                             const __grid_constant__ ChainMaps maps) {
    using Cf = ChainCfg<NS>;
    constexpr int NSLAB = 128 / NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    const uint32_t sbase = tc::smem_u32(smem);
    int* meta = reinterpret_cast<int*>(smem + Cf::OFF_META);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::OFF_BAR);
    uint64_t* bar_p = bars + 0;        // producer: W = T_w K complete
    uint64_t* bar_p2 = bars + 1;       // producer: U~ = T_u V complete
    uint64_t* bar_c1 = bars + 2;       // chain: [Q;W] S over dk 0-63 complete
    uint64_t* bar_c2 = bars + 3;       // chain: [Q;W] S over dk 64-127 complete
    uint64_t* bar_ds = bars + 4;       // chain: K^T U' complete
    uint64_t* bar_y = bars + 5;        // chain: M U complete
    uint64_t* bar_tt = bars + 6;       // T_w, T_u of the next chunk landed in TT
    uint64_t* bar_full = bars + 7;     // [2 slots]
    uint64_t* bar_dsd = bars + 9;      // [2 slots] ds_done
    uint64_t* bar_mfree = bars + 11;   // [2 slots] m_empty
    uint64_t* bar_q = bars + 13;       // [2 slots]
    uint64_t* bar_m = bars + 15;       // [2 slots]
    uint64_t* bar_kv = bars + 17;      // [3 stages] K and V landed (bytes)
    uint64_t* bar_rs = bars + 20;      // [2] the 4 slab CTAs' y^2 sums of a chunk landed (gated, bytes)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::OFF_BAR + 192);
    int* s_base = reinterpret_cast<int*>(smem + Cf::OFF_BAR + 200);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slab = blockIdx.x % NSLAB;
    const int h = (blockIdx.x / NSLAB) % a.H;
    const int n = blockIdx.x / (NSLAB * a.H);
    const int H = a.H;
    int t_begin, t_end;
    seq_bounds(a.cu, n, a.num_seqs, a.N, t_begin, t_end);

    if (warp == 0) {
        const int base = chunks_before(a.cu, a.num_seqs, a.N, n);
        if (lane == 0) *s_base = base;
    }
    if (tid == 0) {
        for (int i = 0; i < Cf::NBARS; ++i) tc::mbar_init(bars + i, 1);
        tc::fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, Cf::TMEM_COLS);
    tc::tc_fence_before();
    __syncthreads();
    if constexpr (GATED) tc::cluster_sync();  // peers' barriers exist before anyone stores to them
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int rec_base = *s_base;
    // malformed cu_seqlens (flagged by seq_bounds) can describe more chunks than the workspace
    // holds: never index past its last record
    const long long rec_end = chunk_count_bound(a.N, a.num_seqs, a.cu != nullptr);
    int nchunks = (t_end - t_begin + kChunk - 1) / kChunk;
    if (rec_base + (long long)nchunks > rec_end) {
        if (tid == 0) raise_error(kErrSeqlens);
        nchunks = (int)max(0LL, rec_end - rec_base);
    }
    const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    auto vec = [&](int b) { return reinterpret_cast<float*>(smem + Cf::OFF_VEC + b * 1024); };
    auto QWoff = [&](int b) { return Cf::OFF_QW + b * 2 * Cf::QW_HALF; };
    auto Koff = [&](int s) { return Cf::OFF_KS + s * 2 * Cf::K_HALF; };
    auto Voff = [&](int s) { return Cf::OFF_VS + s * 64 * Cf::ROWB; };

    if (warp < 4) {
        // =============================== chain group ===================================
        constexpr int BID = 1;
        uint32_t ph_c1 = 0, ph_c2 = 0, ph_ds = 0, ph_y = 0;
        bool ok = true, c1_pending = false, c2_pending = false, ds_pending = false, mu_pending = false;
        // each thread waits for a tcgen05.commit on its own; a timeout flags the error, lets the
        // MMAs drain, and is combined over the group at the next barrier
        auto wait_mma = [&](uint64_t* bar, uint32_t& ph) -> bool {
            const bool w = tc::mbar_wait_bounded(bar, ph, a.budget);
            if (!w) {
                raise_error(kErrTimeout);
                tc::mbar_wait_bounded(bar, ph, 4000000000ull);
            }
            ph ^= 1u;
            tc::tc_fence_after();
            return w;
        };
        // smem operands written by this group become visible to the tensor cores and TMA;
        // returns the AND of v over the group
        auto operands_ready = [&](bool v) -> bool {
            tc::fence_async_smem();
            tc::tc_fence_before();
            const bool all = tc::bar_and(BID, 128, v);
            tc::tc_fence_after();
            return all;
        };
        constexpr uint32_t id_slab = idesc16<BF>(128, NS, false, true);    // [Q;W] S
        constexpr uint32_t id_ds = idesc16<BF>(128, 2 * NS, true, true);   // K^T [U' hi | U' lo]
        constexpr uint32_t id_mu = idesc16<false>(128, NS, false, true);   // M U, both fp16
        // operand descriptors at k-step 0 of slot / stage 0; k-steps and slots are byte offsets
        const uint64_t dQW0 = tc::smem_desc(sbase + Cf::OFF_QW, 16, 1024, tc::kSw128);      // K-major [Q;W]
        const uint64_t dK0 = tc::smem_desc(sbase + Cf::OFF_KS, Cf::K_HALF, 1024, tc::kSw128);  // MN-major K^T
        const uint64_t dM0 = tc::smem_desc(sbase + Cf::OFF_M, 16, 1024, tc::kSw128);
        const uint64_t dSS0 = tc::smem_desc(sbase + Cf::OFF_SS, 128 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
        const uint64_t dSU0 = tc::smem_desc(sbase + Cf::OFF_SU, 64 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
        const uint64_t dSU20 = tc::smem_desc(sbase + Cf::OFF_SU2, 64 * Cf::UROWB, 8 * Cf::UROWB, tc::kSw128);

        const size_t st_base = ((size_t)n * H + h) * 128 * 128 + (size_t)tid * 128 + slab * NS;
        float S[NS];
#pragma unroll
        for (int j = 0; j < NS; j += 4) {
            float4 v4 = a.S0 ? *reinterpret_cast<const float4*>(a.S0 + st_base + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
        }
#pragma unroll
        for (int c = 0; c < NS / 8; ++c) st16(smem + Cf::OFF_SS + tc::swz_off(tid, c, Cf::ROWB), pack8<BF>(S + 8 * c));
        float* nw = reinterpret_cast<float*>(smem + Cf::OFF_NW);
        if (GATED && tid < NS) nw[tid] = 1.f + a.norm_w[slab * NS + tid];
        operands_ready(true);

        // M U of chunk ci (slot bb) -> COL_MU; by thread 0 once M(ci) has landed.  A wait that runs
        // out is flagged and then completed (the copy always lands), so the MMA is always issued
        // and every commit below arrives.
        auto issue_mu = [&](int ci) -> bool {
            bool w = true;
            if (tid == 0) {
                const int bb = ci & 1;
                w = tc::mbar_wait_bounded(bar_m + bb, (ci >> 1) & 1, a.budget);
                if (!w) {
                    raise_error(kErrTimeout);
                    tc::mbar_wait_bounded(bar_m + bb, (ci >> 1) & 1, 4000000000ull);
                }
                const uint64_t am0 = desc_add(dM0, bb * 8192), bu0 = desc_add(dSU0, bb * 64 * Cf::ROWB);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // rows 0-63: M U (rows 64-127 read the next tile: unused)
                    tc::mma_f16(tmem + Cf::COL_MU, desc_add(am0, kk * 32), desc_add(bu0, kk * 16 * Cf::ROWB), id_mu,
                                kk > 0);
                tc::mma_commit(bar_y);
                if constexpr (!GATED) tc::mma_commit(bar_mfree + bb);  // gated: gate_out frees it
            }
            mu_pending = true;
            return w;
        };

        // y of chunk py (warps 0-1): y = scale (Gamma_r (Q S) + M U); a full chunk is staged in
        // swizzled rows for one TMA store, a sequence's last partial chunk goes out with plain stores.
        int py_c0 = 0, py_L = 0;
        float py_g = 0.f;         // its Gamma_r (rows 0-63)
        float qs[NS];             // its (Q S) row (rows 0-63)
        int py_x = -1;            // its index in the sequence (gated: selects buffers and phases)
        bool gated_ok = true;
        // Gated: out = sigmoid(z) y / sqrt(mean_dv(y^2) + eps) (1 + w).  The four slab CTAs of the
        // cluster each hold 32 of the 128 columns of y.  For every chunk each CTA stores every row's
        // partial sum of squares into all four CTAs' shared memory with st.async, whose bytes
        // complete on the receiver's own bar_rs phase (armed by the receiver: 4 x 64 x 4 bytes).
        // y_epilogue sends and keeps y in yt; gate_out, after the next MMA wait, waits for the phase,
        // forms the full mean and gates yt with the z tile the producer loaded beside M.  Every CTA
        // sends and receives exactly nchunks times, also after an error (see the drain below), so
        // no store is still in flight towards a CTA when it exits.
        float yt[NS];
        bool yt_pending = false;
        int n_sent = 0, n_recv = 0;  // chunks sent to the cluster / phases of bar_rs waited for
        constexpr uint32_t RS_TX = NSLAB * 64 * 4;
        auto send_sums = [&](int x, float ss) {  // warps 0-1
            const int bb = x & 1;
            if (tid == 0) tc::mbar_arrive_expect_tx(bar_rs + bb, RS_TX);
            const uint32_t rs = tc::smem_u32(smem + Cf::OFF_RS) + (uint32_t)((bb * 4 + slab) * 64 + tid) * 4;
            const uint32_t br = tc::smem_u32(bar_rs + bb);
#pragma unroll
            for (int p = 0; p < NSLAB; ++p) tc::st_async_f32(tc::mapa(rs, (uint32_t)p), ss, tc::mapa(br, (uint32_t)p));
            n_sent = x + 1;
        };
        auto stage_rows = [&](const float* t, int dt) {  // a finished row -> YS (full chunk) or memory
            if (py_L == kChunk) {
                uint8_t* ys = smem + Cf::OFF_YS;
                if (dt == kF32) {
#pragma unroll
                    for (int cc = 0; cc < NS / 4; ++cc)
                        *reinterpret_cast<float4*>(ys + tc::swz_off(tid, cc, 4 * NS)) =
                            make_float4(t[4 * cc], t[4 * cc + 1], t[4 * cc + 2], t[4 * cc + 3]);
                } else if (dt == kBF16) {
#pragma unroll
                    for (int cc = 0; cc < NS / 8; ++cc) st16(ys + tc::swz_off(tid, cc, 2 * NS), pack8<true>(t + 8 * cc));
                } else {
#pragma unroll
                    for (int cc = 0; cc < NS / 8; ++cc) st16(ys + tc::swz_off(tid, cc, 2 * NS), pack8<false>(t + 8 * cc));
                }
            } else if (tid < py_L) {
                void* dst = reinterpret_cast<uint8_t*>(GATED ? a.out : a.y) +
                            (((size_t)(py_c0 + tid) * H + h) * 128 + slab * NS) * (dt == kF32 ? 4 : 2);
#pragma unroll
                for (int j = 0; j < NS; j += 4) st4(dst, dt, j, make_float4(t[j], t[j + 1], t[j + 2], t[j + 3]));
            }
        };
        // gated, warps 0-1, while M U runs: this row's gate factors sigmoid(z) (1 + w) of chunk py_x
        // -> GZ (row-private, fp32).  Waits for the z tile itself (its own acquire of bar_m).
        auto gz_prep = [&]() {
            if (!GATED || py_L <= 0) return;
            const int bb = py_x & 1;
            if (!tc::mbar_wait_bounded(bar_m + bb, (py_x >> 1) & 1, a.budget)) {
                raise_error(kErrTimeout);
                gated_ok = false;
                return;
            }
            const uint8_t* zs = smem + Cf::OFF_ZS + bb * 64 * Cf::ROWB;
            uint8_t* gz = smem + Cf::OFF_GZ;
#pragma unroll
            for (int cc = 0; cc < NS / 8; ++cc) {
                const uint4 zr = *reinterpret_cast<const uint4*>(zs + tc::swz_off(tid, cc, Cf::ROWB));
                const uint32_t zw[4] = {zr.x, zr.y, zr.z, zr.w};
                float f[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 z2 = a.z_dt == kBF16 ? unpack2<true>(zw[e]) : unpack2<false>(zw[e]);
                    f[2 * e] = __fdividef(nw[8 * cc + 2 * e], 1.f + __expf(-z2.x));
                    f[2 * e + 1] = __fdividef(nw[8 * cc + 2 * e + 1], 1.f + __expf(-z2.y));
                }
                *reinterpret_cast<float4*>(gz + tc::swz_off(tid, 2 * cc, 4 * NS)) = make_float4(f[0], f[1], f[2], f[3]);
                *reinterpret_cast<float4*>(gz + tc::swz_off(tid, 2 * cc + 1, 4 * NS)) = make_float4(f[4], f[5], f[6], f[7]);
            }
        };
        auto y_epilogue = [&]() {
            if (warp < 2 && py_L > 0) {
                float t[NS];
                tc::tmem_ld32(trow + Cf::COL_MU, t);
#pragma unroll
                for (int j = 0; j < NS; ++j) t[j] = a.scale * (py_g * qs[j] + t[j]);
                if constexpr (GATED) {
                    float ss = 0.f;
#pragma unroll
                    for (int j = 0; j < NS; ++j) {
                        ss += t[j] * t[j];
                        yt[j] = t[j];
                    }
                    send_sums(py_x, ss);
                    yt_pending = true;
                } else {
                    stage_rows(t, a.y_dt);
                }
            }
        };
        auto gate_out = [&]() {  // warps 0-1, after y_epilogue; then M slot and z slot are free
            if (!GATED || !yt_pending) return;
            yt_pending = false;
            const int bb = py_x & 1;
            const uint32_t par = (py_x >> 1) & 1;
            const bool w = tc::mbar_wait_bounded(bar_rs + bb, par, a.budget);
            if (w) n_recv = py_x + 1;
            if (!w) {
                raise_error(kErrTimeout);
                gated_ok = false;
            } else {
                const float* rs = reinterpret_cast<const float*>(smem + Cf::OFF_RS) + bb * 4 * 64;
                float tot = 0.f;
#pragma unroll
                for (int p = 0; p < NSLAB; ++p) tot += rs[p * 64 + tid];
                const float inv = rsqrtf(tot / (NS * NSLAB) + a.eps);
                const uint8_t* gz = smem + Cf::OFF_GZ;
#pragma unroll
                for (int cc = 0; cc < NS / 4; ++cc) {
                    const float4 f = *reinterpret_cast<const float4*>(gz + tc::swz_off(tid, cc, 4 * NS));
                    yt[4 * cc] *= inv * f.x;
                    yt[4 * cc + 1] *= inv * f.y;
                    yt[4 * cc + 2] *= inv * f.z;
                    yt[4 * cc + 3] *= inv * f.w;
                }
                stage_rows(yt, a.z_dt);
            }
            tc::bar_sync(4, 64);  // every read of the z slot (gz_prep) is done
            if (tid == 0) tc::mbar_arrive(bar_mfree + bb);
        };
        auto y_store = [&]() {  // after a barrier that follows the staging
            if (tid == 0 && py_L == kChunk) {
                tc::tma_store_3d(&maps.y, slab * NS, h, py_c0, smem + Cf::OFF_YS);
                tc::bulk_commit();
            }
            py_L = 0;
        };
        // wait for M U of the previous chunk (warps 0-1 need it; all threads keep the phase)
        auto wait_mu = [&]() -> bool {
            bool w = true;
            if (warp < 2) w = wait_mma(bar_y, ph_y);
            else ph_y ^= 1u;
            mu_pending = false;
            return w;
        };

        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1, kst = c % 3;
            bool w = tc::mbar_wait_bounded(bar_full + b, (c >> 1) & 1, a.budget);
            w = w && tc::mbar_wait_bounded(bar_q + b, (c >> 1) & 1, a.budget);
            if (!(ok = tc::bar_and(BID, 128, w))) {
                if (tid == 0) raise_error(kErrTimeout);
                break;
            }
            tc::tc_fence_after();
            const float* vb = vec(b);  // gamma[0:64] Gamma[64:128] f[128:192] (g prefetch [192:256])
            const int c0 = meta[2 * b], L = meta[2 * b + 1];
            const float gC = vb[64 + 63];
            const float gR = tid < 64 ? vb[64 + tid] : 0.f;
            const float fR = tid >= 64 ? vb[128 + tid - 64] : 0.f;

            // [Q; -W] S over dk 0-63 (thread 0) is added onto [0; U~] already in COL_U[b]; dk 64-127
            // (thread 32) goes to COL_1B.  Their sum: Q S in lanes 0-63, U = U~ - W S in lanes 64-127.
            if (tid == 0 || tid == 32) {
                const int hf = tid >> 5;
                const uint64_t a0 = desc_add(dQW0, QWoff(b) + hf * Cf::QW_HALF);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16(tmem + (hf ? Cf::COL_1B : Cf::COL_U + b * NS), desc_add(a0, kk * 32),
                                desc_add(dSS0, (hf * 4 + kk) * 16 * Cf::ROWB), id_slab, hf == 0 || kk > 0);
                tc::mma_commit(hf ? bar_c2 : bar_c1);
            }
            c1_pending = c2_pending = true;
            if (c > 0 && warp < 2) gz_prep();  // gated: gate factors of the previous chunk meanwhile
            c1_pending = false;
            const bool w1 = wait_mma(bar_c1, ph_c1);
            c2_pending = false;
            const bool w2 = wait_mma(bar_c2, ph_c2);
            // The previous chunk's M U, then its y (warps 0-1), while warps 2-3 form U: the MMA front
            // end is otherwise idle until the state MMA, so M U delays neither product of the chain.
            bool wm = true, wy = true;
            if (c > 0) {
                wm = issue_mu(c - 1);
                wy = wait_mu();
                if (wy || GATED) y_epilogue();  // gated: the cluster exchange keeps step
            }

            {
                float d1[NS], d2[NS];
                tc::tmem_ld32(trow + Cf::COL_U + b * NS, d1);
                tc::tmem_ld32(trow + Cf::COL_1B, d2);
                if (warp >= 2) {  // U (fp16, for M U), U' = f U (hi + lo, for K^T U')
                    const int r = tid - 64;
                    float ut[NS];
#pragma unroll
                    for (int j = 0; j < NS; ++j) ut[j] = d1[j] + d2[j];
                    uint8_t* su = smem + Cf::OFF_SU + b * 64 * Cf::ROWB;
#pragma unroll
                    for (int cc = 0; cc < NS / 8; ++cc) {
                        uint4 hi, lo;
                        st16(su + tc::swz_off(r, cc, Cf::ROWB), pack8<false>(ut + 8 * cc));
                        float u2[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) u2[e] = fR * ut[8 * cc + e];
                        split8<BF>(u2, hi, lo);
                        st16(smem + Cf::OFF_SU2 + tc::swz_off(r, cc, Cf::UROWB), hi);
                        st16(smem + Cf::OFF_SU2 + tc::swz_off(r, cc + NS / 8, Cf::UROWB), lo);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < NS; ++j) qs[j] = d1[j] + d2[j];
                }
            }
            if (warp < 2) gate_out();
            if (!(ok = operands_ready(wm && wy && w1 && w2 && gated_ok))) break;  // also orders the staged rows
            y_store();

            // K^T U' -> state increment; its completion also releases slot b and K stage kst
            if (tid == 0) {
                const uint64_t ak0 = desc_add(dK0, Koff(kst) - Cf::OFF_KS);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16(tmem + Cf::COL_DS, desc_add(ak0, kk * 2048), desc_add(dSU20, kk * 16 * Cf::UROWB), id_ds, kk > 0);
                tc::mma_commit(bar_ds);
                tc::mma_commit(bar_dsd + b);
            }
            ds_pending = false;
            const bool w3 = wait_mma(bar_ds, ph_ds);

            {
                float t[NS], t2[NS];
                tc::tmem_ld32(trow + Cf::COL_DS, t);
                tc::tmem_ld32(trow + Cf::COL_DS + NS, t2);
#pragma unroll
                for (int j = 0; j < NS; ++j) S[j] = gC * S[j] + (t[j] + t2[j]);
#pragma unroll
                for (int cc = 0; cc < NS / 8; ++cc) st16(smem + Cf::OFF_SS + tc::swz_off(tid, cc, Cf::ROWB), pack8<BF>(S + 8 * cc));
            }
            py_c0 = c0;
            py_L = L;
            py_g = gR;
            py_x = c;
            if (tid == 0) tc::bulk_wait_read0();  // YS is free before the next staging writes it
            if (!(ok = operands_ready(w3))) break;
        }
        if (ok && nchunks > 0) {  // the last chunk's M U and y
            if (warp < 2) gz_prep();
            const bool wm = issue_mu(nchunks - 1);
            const bool wy = wait_mu();
            if (wy || GATED) y_epilogue();
            if (warp < 2) gate_out();
            if ((ok = operands_ready(wm && wy && gated_ok))) y_store();
        }
        // never free TMEM under an MMA in flight
        if (c1_pending) tc::mbar_wait_bounded(bar_c1, ph_c1, 4000000000ull);
        if (c2_pending) tc::mbar_wait_bounded(bar_c2, ph_c2, 4000000000ull);
        if (ds_pending) tc::mbar_wait_bounded(bar_ds, ph_ds, 4000000000ull);
        if (mu_pending) tc::mbar_wait_bounded(bar_y, ph_y, 4000000000ull);
        if (tid == 0) tc::bulk_wait0();
        if (GATED && warp < 2) {
            // the rest of the cluster protocol after an early exit: send the chunks not sent (zeros),
            // then wait for every phase not yet seen -- one phase armed at a time, so each wait's
            // parity is unambiguous, and bytes sent to this CTA all land before it exits
            for (int x = n_recv; x < nchunks; ++x) {
                if (x >= n_sent) send_sums(x, 0.f);
                tc::mbar_wait_bounded(bar_rs + (x & 1), (x >> 1) & 1, 4000000000ull);
            }
        }
        if (ok && a.S_T) {
#pragma unroll
            for (int j = 0; j < NS; j += 4)
                *reinterpret_cast<float4*>(a.S_T + st_base + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    } else {
        // =============================== producer group ================================
        constexpr int BID = 2;
        const int it = tid - 128;
        tc::wait_prerequisites();  // the records of chunk_ut_kernel are complete and visible
        uint32_t ph_w = 0, ph_u = 0;
        bool ok = true;
        constexpr uint32_t id_v = idesc16<false>(128, NS, false, true);  // T_u V in fp16
        constexpr uint32_t id_w = idesc16<BF>(128, 128, false, true);
        const uint64_t dTT0 = tc::smem_desc(sbase + Cf::OFF_TT, 16, 1024, tc::kSw128);
        const uint64_t dV0 = tc::smem_desc(sbase + Cf::OFF_VS, 64 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
        const uint64_t dK0 = tc::smem_desc(sbase + Cf::OFF_KS, Cf::K_HALF, 1024, tc::kSw128);  // MN-major K

        // copies are issued by one thread of warp 6, which has no part in the gate arithmetic
        constexpr int kIssuer = 64;
        // copies in flight into this CTA's shared memory, for the exit drain
        int kv_issued = -1, kv_landed = -1, tt_issued = -1, tt_landed = -1;
        int q_last0 = -1, q_last1 = -1, m_last0 = -1, m_last1 = -1;
        auto rec_ptr = [&](int ci) {
            return reinterpret_cast<const uint8_t*>(a.workspace) + ((size_t)(rec_base + ci) * H + h) * kRecBytes;
        };
        auto issue_kv = [&](int ci) {  // K and the V slab of chunk ci -> stage ci % 3
            kv_issued = ci;
            if (it != kIssuer) return;
            const int c0 = t_begin + ci * kChunk, s = ci % 3;
            uint64_t* bk = bar_kv + s;
            tc::mbar_arrive_expect_tx(bk, Cf::KV_TX);
            tc::tma_load_3d(smem + Koff(s), &maps.k, 0, h, c0, bk);
            tc::tma_load_3d(smem + Koff(s) + Cf::K_HALF, &maps.k, 64, h, c0, bk);
            tc::tma_load_3d(smem + Voff(s), &maps.v, slab * NS, h, c0, bk);
        };
        auto issue_q = [&](int ci) {  // Q of chunk ci -> rows 0-63 of [Q;W] slot ci & 1
            const int bb = ci & 1;
            (bb ? q_last1 : q_last0) = ci;
            if (it != kIssuer) return;
            const int c0 = t_begin + ci * kChunk;
            uint8_t* qw = smem + QWoff(bb);
            tc::mbar_arrive_expect_tx(bar_q + bb, Cf::Q_TX);
            tc::tma_load_3d(qw, &maps.q, 0, h, c0, bar_q + bb);
            tc::tma_load_3d(qw + Cf::QW_HALF, &maps.q, 64, h, c0, bar_q + bb);
        };
        auto issue_m = [&](int ci) {  // M of chunk ci -> M slot ci & 1 (issuer thread only)
            const int bb = ci & 1;
            (bb ? m_last1 : m_last0) = ci;
            tc::mbar_arrive_expect_tx(bar_m + bb, GATED ? Cf::M_TX + Cf::Z_TX : Cf::M_TX);
            tc::bulk_g2s(smem + Cf::OFF_M + bb * 8192, rec_ptr(ci) + kRecM, 8192, bar_m + bb);
            if constexpr (GATED)
                tc::tma_load_3d(smem + Cf::OFF_ZS + bb * 64 * Cf::ROWB, &maps.z, slab * NS, h, t_begin + ci * kChunk,
                                bar_m + bb);
        };
        auto issue_tt = [&](int ci) {  // T_w (twice) and T_u of chunk ci -> TT rows 0-127, 192-255
            tt_issued = ci;
            if (it != kIssuer) return;
            tc::mbar_arrive_expect_tx(bar_tt, 3 * 8192);
            tc::bulk_g2s(smem + Cf::OFF_TT, rec_ptr(ci) + kRecTw, 8192, bar_tt);
            tc::bulk_g2s(smem + Cf::OFF_TT + 8192, rec_ptr(ci) + kRecTw, 8192, bar_tt);
            tc::bulk_g2s(smem + Cf::OFF_TT + 24576, rec_ptr(ci) + kRecTu, 8192, bar_tt);
        };
        // g of chunk ci (beta is already inside T_w, T_u) -> vec(ci & 1)[192:256] by cp.async, two
        // chunks ahead, so no thread waits on the load; one cp.async group per chunk (warps 4-5)
        auto load_gates = [&](int ci) {
            if (it < 64 && ci < nchunks) {
                const int c0 = t_begin + ci * kChunk, L = min(kChunk, t_end - c0);
                const bool in = it < L;
                tc::cp_async4(vec(ci & 1) + 192 + it, in ? a.g + (size_t)(c0 + it) * H + h : a.g, in ? 4u : 0u);
            }
            if (it < 64) tc::cp_async_commit();
        };
        // TT rows 128-191 stay zero: A = [0; T_u] leaves lanes 0-63 of the U~ accumulator at zero
#pragma unroll
        for (int i = 0; i < 4; ++i)
            st16(smem + Cf::OFF_TT + 16384 + (it + 128 * i) * 16, make_uint4(0, 0, 0, 0));
        tc::fence_async_smem();
        if (it == kIssuer) {
            tc::prefetch_tmap(&maps.k);
            tc::prefetch_tmap(&maps.q);
            tc::prefetch_tmap(&maps.v);
            if constexpr (GATED) tc::prefetch_tmap(&maps.z);
        }
        if (nchunks > 0) {
            issue_kv(0);
            issue_tt(0);
        }
        load_gates(0);
        load_gates(1);

        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1, kst = c % 3;
            const int c0 = t_begin + c * kChunk, L = min(kChunk, t_end - c0);
            float* vb = vec(b);
            // slot b, U~ columns b and K stage (c + 1) % 3 are free once the state MMA of c - 2 is done
            bool w = tc::mbar_wait_bounded(bar_dsd + b, ((c >> 1) & 1) ^ 1, a.budget);
            if (!(ok = tc::bar_and(BID, 128, w))) {
                if (it == 0) raise_error(kErrTimeout);
                break;
            }
            issue_q(c);
            if (c + 1 < nchunks) issue_kv(c + 1);

            // ---- gates of chunk c (warps 4-5): gamma (inclusive prefix sum), Gamma,
            //      f = exp(gamma_C - gamma) -----------------------------------------------------------
            if (it < 64) {
                constexpr int BID_G = 3;
                tc::cp_async_wait<1>();  // this chunk's group; the next chunk's may still be in flight
                float gv = vb[192 + it];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, gv, o);
                    if (lane >= o) gv += y;
                }
                vb[it] = gv;
                if (it == 0) {
                    meta[2 * b] = c0;
                    meta[2 * b + 1] = L;
                }
                tc::bar_sync(BID_G, 64);
                if (it >= 32) vb[it] += vb[31];
                tc::bar_sync(BID_G, 64);
                vb[64 + it] = __expf(vb[it]);
                vb[128 + it] = __expf(vb[63] - vb[it]);
            }

            // ---- W = T_w K (thread 0; both lane halves) and U~ = T_u V (thread 32; lanes 64-127),
            //      two issuers with their own commits ---------------------------------------------------
            w = tc::mbar_wait_bounded(bar_kv + kst, (c / 3) & 1, a.budget);
            w = w && tc::mbar_wait_bounded(bar_tt, c & 1, a.budget);
            if (!(ok = tc::bar_and(BID, 128, w))) {
                if (it == 0) raise_error(kErrTimeout);
                break;
            }
            kv_landed = c;
            tt_landed = c;
            if constexpr (BF) {  // V slab bf16 -> fp16 in place (exact for every normal value)
                uint8_t* vs = smem + Voff(kst);
#pragma unroll
                for (int i = 0; i < (64 * Cf::ROWB) / (16 * 128); ++i) {
                    uint4* p16 = reinterpret_cast<uint4*>(vs + (it + 128 * i) * 16);
                    const uint4 u = *p16;
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
                    uint32_t o4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = unpack2<true>(w4[e]);
                        o4[e] = pack2<false>(f.x, f.y);
                    }
                    *p16 = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                }
                tc::fence_async_smem();
                tc::bar_sync(BID, 128);
            }
            tc::tc_fence_after();
            if (it == 0) {
                const uint64_t bk0 = desc_add(dK0, Koff(kst) - Cf::OFF_KS);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16(tmem + Cf::COL_W, desc_add(dTT0, kk * 32), desc_add(bk0, kk * 2048), id_w, kk > 0);
                tc::mma_commit(bar_p);
            } else if (it == 32) {  // [0; T_u] V (fp16): lanes 0-63 zero, lanes 64-127 U~
                const uint64_t bv0 = desc_add(dV0, Voff(kst) - Cf::OFF_VS);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16(tmem + Cf::COL_U + b * NS, desc_add(dTT0, 16384 + kk * 32),
                                desc_add(bv0, kk * 16 * Cf::ROWB), id_v, kk > 0);
                tc::mma_commit(bar_p2);
            }
            bool ww = tc::mbar_wait_bounded(bar_p, ph_w, a.budget);
            if (!ww) {
                raise_error(kErrTimeout);
                tc::mbar_wait_bounded(bar_p, ph_w, 4000000000ull);
            }
            ph_w ^= 1u;
            bool wu = tc::mbar_wait_bounded(bar_p2, ph_u, a.budget);
            if (!wu) {
                raise_error(kErrTimeout);
                tc::mbar_wait_bounded(bar_p2, ph_u, 4000000000ull);
            }
            ph_u ^= 1u;
            tc::tc_fence_after();
            if (!(ok = tc::bar_and(BID, 128, ww && wu))) break;
            if (c + 1 < nchunks) issue_tt(c + 1);  // the MMAs have read TT

            // ---- -W -> rows 64-127 of [Q; -W] in slot b: lanes 0-63 write columns 0-63, lanes 64-127
            //      columns 64-127 (each lane half of the accumulator holds all of W) ------------------
            {
                const int r = it & 63, hf = it >> 6;
                float wv[64];
                tc::tmem_ld32(trow + Cf::COL_W + 64 * hf, wv);
                tc::tmem_ld32(trow + Cf::COL_W + 64 * hf + 32, wv + 32);
#pragma unroll
                for (int j = 0; j < 64; ++j) wv[j] = -wv[j];
                uint8_t* qw = smem + QWoff(b) + hf * Cf::QW_HALF;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) st16(qw + tc::swz_off(64 + r, cc, 128), pack8<BF>(wv + 8 * cc));
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::bar_sync(BID, 128);
            if (it == 0) tc::mbar_arrive(bar_full + b);  // hand chunk c to the chain group

            // ---- M of chunk c, once M U of c - 2 has read the slot ---------------------------------
            if (it == kIssuer) {
                if (tc::mbar_wait_bounded(bar_mfree + b, ((c >> 1) & 1) ^ 1, a.budget)) issue_m(c);
                else raise_error(kErrTimeout);
            }
            load_gates(c + 2);
        }
        if (it < 64) tc::cp_async_wait<0>();  // no copy into shared memory left in flight
        // never leave with copies into this CTA's shared memory in flight
        if (kv_issued > kv_landed) tc::mbar_wait_bounded(bar_kv + kv_issued % 3, (kv_issued / 3) & 1, 4000000000ull);
        if (kv_issued > kv_landed + 1)
            tc::mbar_wait_bounded(bar_kv + (kv_issued - 1) % 3, ((kv_issued - 1) / 3) & 1, 4000000000ull);
        if (tt_issued > tt_landed) tc::mbar_wait_bounded(bar_tt, tt_issued & 1, 4000000000ull);
        if (q_last0 >= 0) tc::mbar_wait_bounded(bar_q + 0, (q_last0 >> 1) & 1, 4000000000ull);
        if (q_last1 >= 0) tc::mbar_wait_bounded(bar_q + 1, (q_last1 >> 1) & 1, 4000000000ull);
        if (m_last0 >= 0) tc::mbar_wait_bounded(bar_m + 0, (m_last0 >> 1) & 1, 4000000000ull);
        if (m_last1 >= 0) tc::mbar_wait_bounded(bar_m + 1, (m_last1 >> 1) & 1, 4000000000ull);
        (void)ok;
    }

    if constexpr (GATED) tc::cluster_sync();  // no CTA leaves while a peer may still write to it
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, Cf::TMEM_COLS);
    }
}

template <bool BF>
inline cudaError_t chunk_tc_launch_t(const ChunkArgs& a, const ChainMaps& maps, cudaStream_t st) {
    constexpr int NS = 32;
    using Ch = ChainCfg<NS>;
    cudaError_t e = cudaFuncSetAttribute(chunk_ut_kernel<BF>, cudaFuncAttributeMaxDynamicSharedMemorySize, UtCfg::BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_chain_kernel<NS, BF, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, Ch::BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_chain_kernel<NS, BF, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, Ch::BYTES);
    if (e != cudaSuccess) return e;
    const long long nvc = chunk_count_bound(a.N, a.num_seqs, a.cu != nullptr);
    if (nvc > 0) {
        LaunchScope timed(st, "chunk_ut_kernel");
        chunk_ut_kernel<BF><<<(unsigned)(nvc * a.H), 128, UtCfg::BYTES, st>>>(a, maps);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const unsigned grid = (unsigned)(a.num_seqs * a.H * (128 / NS));
    // Programmatic dependent launch: the chain's prologue overlaps the tail of chunk_ut_kernel;
    // its producer waits for that grid before reading a record.  Gated: the 128 / NS slab CTAs
    // of a (sequence, head) form one cluster.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = Ch::BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 128 / NS;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    if (a.out == nullptr) {
        cfg.numAttrs = 1;
        LaunchScope timed(st, "chunk_chain_kernel");
        return cudaLaunchKernelEx(&cfg, chunk_chain_kernel<NS, BF, false>, a, maps);
    }
    cfg.numAttrs = 2;
    LaunchScope timed(st, "chunk_chain_gated_kernel");
    return cudaLaunchKernelEx(&cfg, chunk_chain_kernel<NS, BF, true>, a, maps);
}

// Both kernels of the chunked path on stream st.  *why is set (and nothing launched) when the
// configuration is not built or a tensor map cannot be encoded.
inline cudaError_t chunk_tc_launch(const ChunkArgs& a, cudaStream_t st, const char** why) {
    *why = nullptr;
    if (a.chunk != kChunk) {
        *why = "only chunk = 64 is built";
        return cudaSuccess;
    }
    constexpr int NS = 32;
    // y (or out) tiles are NS columns = 64 B (16-bit) or 128 B (fp32) per row, stored with the
    // matching swizzle; the gated variant stores out and loads z slabs
    const bool gated = a.out != nullptr;
    const int st_dt = gated ? a.z_dt : a.y_dt;
    const CUtensorMapSwizzle yswz = st_dt == kF32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    ChainMaps maps = {};  // the z map stays empty without the gate
    if (!encode_map_3d(&maps.k, a.k, a.in_dt, a.N, a.H, 128, 64, kChunk, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map_3d(&maps.q, a.q, a.in_dt, a.N, a.H, 128, 64, kChunk, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map_3d(&maps.v, a.v, a.in_dt, a.N, a.H, 128, NS, kChunk, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_map_3d(&maps.y, gated ? a.out : a.y, st_dt, a.N, a.H, 128, NS, kChunk, yswz) ||
        (gated && !encode_map_3d(&maps.z, a.z, a.z_dt, a.N, a.H, 128, NS, kChunk, CU_TENSOR_MAP_SWIZZLE_64B))) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaSuccess;
    }
    return a.in_dt == kBF16 ? chunk_tc_launch_t<true>(a, maps, st) : chunk_tc_launch_t<false>(a, maps, st);
}

}  // namespace gdn
