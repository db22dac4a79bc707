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
//   chunk_ut_kernel     one CTA per (chunk, head), fully parallel, two CTAs per SM.
//                       [K;Q] K^T on tcgen05 (the 16-bit inputs used directly as operands),
//                       the decay masks, and the unit-lower-triangular inverse T in fp32 on the
//                       CUDA cores; then one N = 256 product [T_w; T_u] [K | V] with
//                       T_w = T diag(beta Gamma) and T_u = T diag(beta) gives W = T_w K and
//                       U~ = T_u V.  Writes a 40.5 KB record per (chunk, head): -W and M in the
//                       128B-swizzled operand layout and U~ as four 32-column slabs, all fp16,
//                       and the chunk's gates Gamma_r and Gamma_C / Gamma_r in fp32.
//   chunk_chain_kernel  one CTA per (sequence, head, 32-column dv slab), sequential over
//                       the chunks.  A producer warpgroup only copies: each chunk's K and Q by
//                       TMA, -W, U~, M and the gates from the record by bulk copies, straight into
//                       operand slots (bf16 K and Q converted to fp16 in place), one chunk ahead
//                       of the chain.  A chain warpgroup
//                       carries the fp32 state (one row per thread) through two dependent
//                       tensor-core round trips per chunk:
//                           [Q; -W] S        -> Q S and -W S, so U = U~ - W S
//                           K^T U'           -> S' = Gamma_C S + K^T U'
//                       with U' = diag(Gamma_C / Gamma) U, while M U, for
//                       Y = Gamma (Q S) + M U, is issued once the next chunk's [Q; -W] S
//                       has completed, when the MMA front end is otherwise idle.  Sixteen MMA
//                       instructions per chunk, none of them in the producer.
//                       Q/W/M/U~ slots are double-buffered, K stages triple-buffered, all
//                       handed over with mbarriers; full chunks of y leave through swizzled
//                       TMA stores.  It is launched as a programmatic dependent of
//                       chunk_ut_kernel.  The gated variant applies eq. (11)'s output gate
//                       in the y epilogue, the four slab CTAs of a (sequence, head) forming
//                       one cluster that exchanges row sums of squares.
// Operands are 16-bit with fp32 accumulation in TMEM.  A tcgen05.mma instruction with
// M = 128 costs the SM's MMA pipe about 95 cycles for any N up to 64 (N = 128: about 147,
// N = 256: about 173, measured), so products are shaped to use few instructions, and the
// per-(chunk, head) products are formed once in chunk_ut_kernel rather than once per slab.
// bf16 inputs must lie inside the fp16 range (|x| < 65504), as unit-norm keys and queries do.  [K;Q] K^T reads q and k exactly as stored.  Every product of the
// chain runs on fp16 operands (11 significant bits): bf16 q, k and v are converted to fp16 in
// shared memory when they land (exact for |x| >= 2^-14), and their partners T_w, W, S and U'
// are formed in fp16.  bf16 partners (8 bits) would let the error of a row whose y is small
// exceed the bound once eq. (11) normalises that row.  U' = f U enters as one fp16 value (the
// state's error stays near 5e-4 of its scale, well inside the bound).
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
#include "warp_mma.cuh"

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

// TMA descriptors of both kernels: [N, H, 128] views of k, q and v (64-column halves, 128B
// swizzle), z (NS-column slab, 64B swizzle) and y -- or out, when the gate is fused --
// (NS-column slab stores, swizzled to the row width).
struct ChainMaps {
    CUtensorMap k, q, v, y, z;
};

constexpr int kChunk = 64;
// Record of one (chunk, head), written by chunk_ut_kernel, all fp16:
constexpr int kRecW = 0;           // -W: two dk halves, each [64 rows x 128 B] 128B-swizzled K-major,
                                   // ready to be rows 64-127 of the chain's [Q; -W] operand
constexpr int kRecM = 16384;       // M: [64 rows x 128 B] 128B-swizzled K-major
constexpr int kRecU = 24576;       // U~: four 32-column dv slabs, each [64 rows x 64 B] row-major
constexpr int kRecUSlab = 4096;
constexpr int kRecG = 40960;       // Gamma_r = exp(gamma_r) [64] then f_r = exp(gamma_C - gamma_r) [64], fp32
constexpr int kRecBytes = 41472;

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

template <bool BF>
__host__ __device__ constexpr uint32_t idesc16(int M, int N, bool a_mn, bool b_mn) {
    return BF ? tc::idesc_bf16(M, N, a_mn, b_mn) : tc::idesc_f16(M, N, a_mn, b_mn);
}

__device__ __forceinline__ void st16(uint8_t* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

// BYTES (a multiple of 16 * NT) of bf16 values at p rewritten as fp16, 16 bytes per thread per
// pass over NT threads (it = the thread's index among them), every load issued before the first
// conversion.
template <int NT, int BYTES>
__device__ __forceinline__ void to_f16_block(uint8_t* p, int it) {
    static_assert(BYTES % (16 * NT) == 0, "whole passes");
    constexpr int ITER = BYTES / (16 * NT);
    uint4 u[ITER];
#pragma unroll
    for (int k = 0; k < ITER; ++k) u[k] = *reinterpret_cast<const uint4*>(p + (it + k * NT) * 16);
#pragma unroll
    for (int k = 0; k < ITER; ++k) {
        const uint32_t w4[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
        uint32_t o4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = unpack2<true>(w4[e]);
            o4[e] = pack2<false>(f.x, f.y);
        }
        *reinterpret_cast<uint4*>(p + (it + k * NT) * 16) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
}

// =====================================================================================
// chunk_ut_kernel: per (chunk, head) -- masks and the UT transform
// =====================================================================================

struct UtCfg {
    static constexpr int THREADS = 256;
    static constexpr int LD = 68;                           // fp32 row stride of A and T
    // [K h0 | Q h0 | K h1 | Q h1 | V h0 | (gap) | V h1], 8 KB tiles [64 rows x 128 B], 128B
    // swizzle.  [K_h; Q_h] is the A operand of half h of [K;Q] K^T; K h0, K h1, V h0, V h1 sit
    // 16 KB apart, the column-block stride of the MN-major B operand [K | V] (N = 256).
    static constexpr int OFF_K = 0, OFF_Q = 8192, OFF_V = 32768, KV_LBO = 16384;
    // fp32 scratch of the block inverse over Q h0 once [K;Q] K^T has read it: the level-one
    // products [2 blocks][16][LDX1] and the level-two product [32][LDX2]
    static constexpr int OFF_X1 = 8192, LDX1 = 20, OFF_X2 = OFF_X1 + 2 * 16 * LDX1 * 4, LDX2 = 36;
    static constexpr int OFF_VEC = 40960;                   // gamma, Gamma, beta, colf: 4 x 64 (gap)
    static constexpr int OFF_META = OFF_VEC + 1024;
    static constexpr int OFF_BAR = OFF_META + 32;
    static constexpr int OFF_A = 57344;                     // fp32 A [64][LD]; later [T_w; T_u]
    static constexpr int OFF_TOP = OFF_A;                   //   fp16 [128 rows x 128 B], 128B swizzle
    static constexpr int OFF_T = OFF_A + 64 * LD * 4;       // fp32 T [64][LD]
    static constexpr int BYTES = OFF_T + 64 * LD * 4 + 1024;
    static_assert(OFF_BAR + 64 <= OFF_V + 16384, "vectors and barriers fit in the gap");
    static_assert(OFF_X2 + 32 * LDX2 * 4 <= 16384, "inverse scratch fits in Q h0");
    static_assert(64 * LD * 4 >= 16384 && OFF_A % 1024 == 0, "[T_w; T_u] fits over A");
    static constexpr uint32_t TMEM_COLS = 256;              // [K;Q] K^T (cols 0-63), then [T_w;T_u][K|V]
};

// One CTA (eight warps) per (chunk, head): the UT transform of the chunk and the products that
// depend on it alone.  [K;Q] K^T gives A and M; T = (I + A)^-1 in fp32 (16x16 diagonal blocks by
// forward substitution on the CUDA cores, the off-diagonal blocks by recursive doubling,
//     T21 = -T22 A21 T11   for 16x16 blocks, then the same for the 32x32 halves,
// as warp-level mma.sync products of fp32 values split into fp16 pairs); then one N = 256
// product
//     [T_w; T_u] [K | V]  ->  lanes 0-63: W = T_w K (columns 0-127),
//                             lanes 64-127: U~ = T_u V (columns 128-255)
// (the other two blocks are not used), with T_w = T diag(beta Gamma), T_u = T diag(beta), K and
// V converted to fp16 once [K;Q] K^T has read them.  -W, M and U~ go to the record in fp16.
template <bool BF>
__global__ void __launch_bounds__(UtCfg::THREADS, 2) chunk_ut_kernel(const __grid_constant__ ChunkArgs a,
                                                                     const __grid_constant__ ChainMaps maps) {
    using Cf = UtCfg;
    constexpr int LD = Cf::LD, NT = Cf::THREADS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    const uint32_t sbase = tc::smem_u32(smem);
    float* fA = reinterpret_cast<float*>(smem + Cf::OFF_A);
    float* fT = reinterpret_cast<float*>(smem + Cf::OFF_T);
    float* fX1 = reinterpret_cast<float*>(smem + Cf::OFF_X1);
    float* fX2 = reinterpret_cast<float*>(smem + Cf::OFF_X2);
    float* vb = reinterpret_cast<float*>(smem + Cf::OFF_VEC);  // gamma[0:64] Gamma[64:128] beta[128:192] colf[192:256]
    int* meta = reinterpret_cast<int*>(smem + Cf::OFF_META);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cf::OFF_BAR);       // MMA done (two phases)
    uint64_t* bar_ld = bar + 1;                                            // K, Q, V tiles landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::OFF_BAR + 16);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // TMEM lane quadrant and column half of this warp in the epilogues (two warps per quadrant)
    const int quad = warp & 3, chalf = warp >> 2;
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

    // ---- K, Q, V as they are stored (bf16 or fp16), by TMA into the 128B-swizzled operand
    //      layout.  Rows past the sequence end hold other tokens (or the fill of a load past N);
    //      they only meet beta = 0 or the strictly-upper mask, so nothing needs clearing. ---------
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(bar_ld, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(bar_ld, 6 * 8192);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tc::tma_load_3d(smem + Cf::OFF_K + hf * 16384, &maps.k, 64 * hf, h, t0, bar_ld);
            tc::tma_load_3d(smem + Cf::OFF_Q + hf * 16384, &maps.q, 64 * hf, h, t0, bar_ld);
            tc::tma_load_3d(smem + Cf::OFF_V + hf * Cf::KV_LBO, &maps.v, 64 * hf, h, t0, bar_ld);
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
        // the chain's gates of this chunk: Gamma_r and f_r = exp(gamma_C - gamma_r) (positions past
        // the sequence end carry g = 0, so gamma_C = gamma of the last token)
        float* rg = reinterpret_cast<float*>(rec + kRecG);
        rg[tid] = vb[64 + tid];
        rg[64 + tid] = __expf(vb[63] - vb[tid]);
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

    // ---- [K;Q] K^T (the inputs' own format) -------------------------------------------------------
    if (tid == 0 && landed) {
        constexpr uint32_t id = idesc16<BF>(128, 64, false, false);
        const uint64_t d0 = tc::smem_desc(sbase + Cf::OFF_K, 16, 1024, tc::kSw128);
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

    bool done2 = false;
    if (landed && done) {
        // ---- masks: A (fp32) for the solve; M (fp16) straight into the record.  TMEM lane
        //      32 quad + lane is row r of [K;Q] K^T, this warp takes columns 32 chalf .. +31 -----------
        {
            float x[32];
            tc::tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + 32 * chalf, x);
            const int r = (32 * quad + lane) & 63, R = r >> 4, rl = r & 15;
            const float gr = vb[r];
            const bool isA = quad < 2;
            const float sc = isA ? vb[128 + r] : 1.f;
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                const int S = 2 * chalf + blk;
                // blocks before the row's own: exp(gamma_r - gamma_e) exp(gamma_e - gamma_s), both <= 1
                const float rowf = S < R ? __expf(gr - vb[16 * S + 15]) : 0.f;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int s = 16 * S + e;
                    float f = rowf * vb[192 + s];
                    if (S == R) f = (isA ? e < rl : e <= rl) ? __expf(gr - vb[s]) : 0.f;
                    x[16 * blk + e] *= sc * f;
                }
            }
            if (isA) {
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4)
                    sts4(fA + r * LD + 32 * chalf + 4 * c4, make_float4(x[4 * c4], x[4 * c4 + 1], x[4 * c4 + 2], x[4 * c4 + 3]));
            } else {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) st16(rec + kRecM + tc::swz_off(r, 4 * chalf + cc, 128), pack8<false>(x + 8 * cc));
            }
        }
        // K and V to fp16 in place for the second product (exact for |x| >= 2^-14); [K;Q] K^T
        // has completed, so nothing reads them meanwhile
        if constexpr (BF) {
            to_f16_block<NT, 8192>(smem + Cf::OFF_K, tid);
            to_f16_block<NT, 8192>(smem + Cf::OFF_K + 16384, tid);
            to_f16_block<NT, 8192>(smem + Cf::OFF_V, tid);
            to_f16_block<NT, 8192>(smem + Cf::OFF_V + Cf::KV_LBO, tid);
        }
        tc::tc_fence_before();
        __syncthreads();

        // ---- T = (I + A)^-1.  16x16 diagonal blocks by forward substitution (warps 0-3, lane =
        //      column); the zeros above each diagonal are written too ---------------------------
        if (warp < 4 && lane < 16) {
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
        // level one (warps 0-3): T_i,i-1 = -T_ii (A_i,i-1 T_i-1,i-1) for i = 1, 3, one 8-column
        // tile per warp
        if (warp < 4) {
            const int bi = warp >> 1, nt = warp & 1, i = 2 * bi + 1, j = i - 1;
            uint32_t ah[4], al[4], bh[2], bl[2];
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            wm::load_a(fA, LD, 16 * i, 16 * j, 1.f, ah, al);
            wm::load_b(fT, LD, 16 * j, 16 * j + 8 * nt, bh, bl);
            wm::mma_split(d, ah, al, bh, bl);
            float* x1 = fX1 + bi * 16 * Cf::LDX1;
            wm::store_c(x1, Cf::LDX1, 0, 8 * nt, d);
            __syncwarp();
            float e[4] = {0.f, 0.f, 0.f, 0.f};
            wm::load_a(fT, LD, 16 * i, 16 * i, -1.f, ah, al);
            wm::load_b(x1, Cf::LDX1, 0, 8 * nt, bh, bl);
            wm::mma_split(e, ah, al, bh, bl);
            wm::store_c(fT, LD, 16 * i, 16 * j + 8 * nt, e);
        }
        __syncthreads();
        // level two (all warps): X = A[32:64, 0:32] T[0:32, 0:32], then T[32:64, 0:32] = -T[32:64,
        // 32:64] X; one 16x8 tile per warp, skipping the zero upper-right 16x16 blocks
        {
            const int mt = warp >> 2, nt = warp & 3;
            uint32_t ah[4], al[4], bh[2], bl[2];
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kt = 0; kt < 2; ++kt) {
                if (kt == 0 && nt >= 2) continue;  // T[0:16, 16:32] = 0
                wm::load_a(fA, LD, 32 + 16 * mt, 16 * kt, 1.f, ah, al);
                wm::load_b(fT, LD, 16 * kt, 8 * nt, bh, bl);
                wm::mma_split(d, ah, al, bh, bl);
            }
            wm::store_c(fX2, Cf::LDX2, 16 * mt, 8 * nt, d);
            __syncthreads();
            float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kt = 0; kt < 2; ++kt) {
                if (mt == 0 && kt == 1) continue;  // T[32:48, 48:64] = 0
                wm::load_a(fT, LD, 32 + 16 * mt, 32 + 16 * kt, -1.f, ah, al);
                wm::load_b(fX2, Cf::LDX2, 16 * kt, 8 * nt, bh, bl);
                wm::mma_split(e, ah, al, bh, bl);
            }
            wm::store_c(fT, LD, 32 + 16 * mt, 8 * nt, e);
        }
        __syncthreads();
        // ---- [T_w; T_u] (fp16) over A: T_w = T diag(beta Gamma) in rows 0-63, T_u = T diag(beta)
        //      in rows 64-127, K-major with K = the chunk position s --------------------------------
        uint8_t* top = smem + Cf::OFF_TOP;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int idx = tid + NT * u, which = idx >> 9, r = (idx >> 3) & 63, cc = idx & 7;
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
            st16(top + tc::swz_off(64 * which + r, cc, 128), pack8<false>(t8));
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();

        // ---- [T_w; T_u] [K | V] -> TMEM columns 0-255 (fp16, N = 256, four k-steps) ------------
        if (tid == 0) {
            constexpr uint32_t id = idesc16<false>(128, 256, false, true);
            const uint64_t da = tc::smem_desc(sbase + Cf::OFF_TOP, 16, 1024, tc::kSw128);
            const uint64_t db = tc::smem_desc(sbase + Cf::OFF_K, Cf::KV_LBO, 1024, tc::kSw128);  // MN-major
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc::mma_f16(tmem, desc_add(da, kk * 32), desc_add(db, kk * 2048), id, kk > 0);
            tc::mma_commit(bar);
        }
        done2 = tc::mbar_wait_bounded(bar, 1, a.budget);
        if (!done2) {
            raise_error(kErrTimeout);
            tc::mbar_wait_bounded(bar, 1, 4000000000ull);
        }
        tc::tc_fence_after();
        if (done2) {
            // quadrants 0-1: -W row r, columns 64 chalf .. +63 -> dk half chalf of the record;
            // quadrants 2-3: U~ row r, columns 128 + 64 chalf .. +63 -> dv slabs 2 chalf, 2 chalf + 1
            const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
            const int r = (32 * quad + lane) & 63;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float x[32];
                tc::tmem_ld32(trow + (quad < 2 ? 0 : 128) + 64 * chalf + 32 * q, x);
                if (quad < 2) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] = -x[e];
                    uint8_t* dst = rec + kRecW + chalf * 8192;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) st16(dst + tc::swz_off(r, 4 * q + cc, 128), pack8<false>(x + 8 * cc));
                } else {
                    uint8_t* dst = rec + kRecU + (2 * chalf + q) * kRecUSlab + r * 64;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) st16(dst + 16 * cc, pack8<false>(x + 8 * cc));
                }
            }
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
    static constexpr uint32_t SWZ = NS == 32 ? tc::kSw64 : tc::kSw128;
    static constexpr int QW_HALF = 128 * 128;                  // one 64-column half of [Q;W]
    static constexpr int K_HALF = 64 * 128;                    // one 64-column half of K
    static constexpr int OFF_QW = 0;                           // [3 stages] [Q;-W]: 2 halves x [128 x 128 B]
    static constexpr int OFF_M = OFF_QW + 3 * 2 * QW_HALF;     // [2 slots] M fp16: [64 x 128 B]
    static constexpr int OFF_KS = OFF_M + 2 * 8192;            // [3 stages] K: 2 halves x [64 x 128 B]
    static constexpr int OFF_UT = OFF_KS + 3 * 2 * K_HALF;     // [3 stages] U~ slab fp16 [64 x ROWB], row-major
    static constexpr int OFF_SS = OFF_UT + 3 * 64 * ROWB;      // S [128 x ROWB]
    static constexpr int OFF_SU = OFF_SS + 128 * ROWB;         // [2 slots] U fp16: [64 x ROWB]
    static constexpr int OFF_SU2 = OFF_SU + 2 * 64 * ROWB;     // U' = f U fp16: [64 x ROWB]
    static constexpr int OFF_YS = OFF_SU2 + 64 * ROWB;         // y rows for the TMA store [64 x NS x 4 B]
    static constexpr int OFF_ZS = OFF_YS + 64 * NS * 4;        // [2 slots] z slab [64 x ROWB] (gated)
    static constexpr int OFF_GZ = OFF_ZS + 2 * 64 * ROWB;      // sigmoid(z) (1 + w) rows, fp32 [64 x NS] (gated)
    static constexpr int OFF_GT = OFF_GZ + 64 * NS * 4;        // [3 stages] Gamma [64], f [64] fp32 (record)
    static constexpr int OFF_RS = OFF_GT + 3 * 512;            // [2] [4 slabs] [64 rows] y^2 sums (gated)
    static constexpr int OFF_NW = OFF_RS + 2 * 4 * 64 * 4;     // 1 + norm_w of this slab (gated)
    static constexpr int OFF_BAR = OFF_NW + NS * 4;
    static constexpr int NBARS = 22;
    static constexpr int BYTES = OFF_BAR + 256 + 1024;
    static constexpr uint32_t K_TX = 2 * K_HALF;               // K of one chunk
    static constexpr uint32_t OP_TX = 2 * 8192 + 2 * 8192 + 64 * ROWB + 512;  // Q, -W, the U~ slab, gates
    static constexpr uint32_t M_TX = 8192;                     // M of one chunk
    static constexpr uint32_t Z_TX = 64 * ROWB;                // z slab of one chunk (gated)
    // TMEM columns; the products of chunk c that y of c needs stay until chunk c + 1 reads them
    static constexpr uint32_t COL_U = 0;                       // [2 slots] x NS: [Q; -W] S over dk 0-63
    static constexpr uint32_t COL_1B = COL_U + 2 * NS;         // [2 slots] x NS: [Q; -W] S over dk 64-127
    static constexpr uint32_t COL_MU = COL_1B + 2 * NS;        // [2 slots] x NS: M U (lanes 0-63)
    static constexpr uint32_t COL_DS = COL_MU + 2 * NS;        // NS: K^T U' 
    static constexpr uint32_t TMEM_COLS = 256;
    static_assert(COL_DS + 2 * NS <= TMEM_COLS, "TMEM budget");
    static_assert(NS == 32, "slab operand rows are one 64-byte swizzle atom");
    static_assert(NBARS * 8 <= 192, "barrier area");
    static_assert(BYTES <= 232448, "shared memory budget");
    static_assert(OFF_M % 1024 == 0 && OFF_KS % 1024 == 0 && OFF_YS % 1024 == 0 && OFF_UT % 1024 == 0 &&
                      OFF_SS % 1024 == 0 && OFF_SU % 1024 == 0 && OFF_SU2 % 1024 == 0 && OFF_ZS % 1024 == 0 &&
                      OFF_GZ % 1024 == 0,
                  "swizzle atoms");
};

// Synchronisation of one chunk c, in stage s = c % 3 for Q, -W, U~ and K, and slot b = c & 1 for M
// and the hand-over:
//   producer -> chain   full[b]      Q(c) and -W(c) in [Q;-W] stage s, U~(c) in U~ stage s, K(c) in
//                                    K stage s (all fp16), gates and bounds of c
//                       m[b]         M(c) landed (bulk copy bytes)
//   chain -> producer   ds_done[s]   the state MMA of c completed: the [Q;-W], U~ and K stages s are
//                                    free (everything else of c was read before); the producer
//                                    refills them with chunk c + 3, two chain periods ahead of use
//                       m_empty[b]   M U of c completed: M slot b and U slot b are free
// The chain issues M U of chunk c once chunk c + 1's [Q;-W] S has completed (the MMA front end is
// idle while warps 2-3 form U) and forms y of c meanwhile.
template <int NS, bool BF, bool GATED>
__global__ void __launch_bounds__(256, 1) chunk_chain_kernel(const __grid_constant__ ChunkArgs a,
                                                             const __grid_constant__ ChainMaps maps) {
    using Cf = ChainCfg<NS>;
    constexpr int NSLAB = 128 / NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    const uint32_t sbase = tc::smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::OFF_BAR);
    uint64_t* bar_c1 = bars + 0;       // chain: [Q;-W] S over dk 0-63 complete
    uint64_t* bar_c2 = bars + 1;       // chain: [Q;-W] S over dk 64-127 complete
    uint64_t* bar_ds = bars + 2;       // chain: K^T U' complete
    uint64_t* bar_y = bars + 3;        // chain: M U complete
    uint64_t* bar_full = bars + 4;     // [2 slots]
    uint64_t* bar_dsd = bars + 6;      // [3 stages] ds_done
    uint64_t* bar_mfree = bars + 9;    // [2 slots] m_empty
    uint64_t* bar_q = bars + 11;       // [3 stages] Q, -W and U~ of a chunk landed (bytes)
    uint64_t* bar_m = bars + 14;       // [2 slots]
    uint64_t* bar_kv = bars + 16;      // [3 stages] K landed (bytes)
    uint64_t* bar_rs = bars + 19;      // [2] the 4 slab CTAs' y^2 sums of a chunk landed (gated, bytes)
    uint64_t* bar_drain = bars + 21;   // every MMA of the three issuing threads completed (exit)
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
        for (int i = 0; i < Cf::NBARS; ++i) tc::mbar_init(bars + i, i == 21 ? 3 : 1);
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
    auto gates = [&](int s) { return reinterpret_cast<const float*>(smem + Cf::OFF_GT + s * 512); };
    auto QWoff = [&](int b) { return Cf::OFF_QW + b * 2 * Cf::QW_HALF; };
    auto Koff = [&](int s) { return Cf::OFF_KS + s * 2 * Cf::K_HALF; };

    if (warp < 4) {
        // =============================== chain group ===================================
        // Per chunk c (slot b = c & 1, stage kst = c % 3):
        //   thread 0 / 32   [Q; -W] S(c) over the two dk halves -> COL_U[b], COL_1B[b]; thread 0 then
        //                   issues M U(c - 1) -> COL_MU[(c - 1) & 1] behind it
        //   warps 2-3       U = U~ - W S (lanes 64-127) -> U (fp16) and U' = f U (fp16); thread 64
        //                   issues K^T U'(c) as soon as these two warps have written U'
        //   warps 0-1       meanwhile y of chunk c - 1 = scale (Gamma (Q S) + M U), all three
        //                   products read from TMEM, staged and stored
        //   all             S = Gamma_C S + K^T U' (one dk row per thread) -> fp16 S operand
        // so the state's critical path holds two MMA round trips and the U epilogue, and the y
        // work of warps 0-1 overlaps it.
        constexpr int BID = 1, BID_U = 5, BID_Y = 4;
        uint32_t ph_c1 = 0, ph_c2 = 0, ph_ds = 0, ph_y = 0;
        bool ok = true;
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
        constexpr uint32_t id_slab = idesc16<false>(128, NS, false, true);    // [Q;W] S
        constexpr uint32_t id_ds = idesc16<false>(128, NS, true, true);       // K^T U' 
        constexpr uint32_t id_mu = idesc16<false>(128, NS, false, true);   // M U, both fp16
        // operand descriptors at k-step 0 of slot / stage 0; k-steps and slots are byte offsets
        const uint64_t dQW0 = tc::smem_desc(sbase + Cf::OFF_QW, 16, 1024, tc::kSw128);      // K-major [Q;W]
        const uint64_t dK0 = tc::smem_desc(sbase + Cf::OFF_KS, Cf::K_HALF, 1024, tc::kSw128);  // MN-major K^T
        const uint64_t dM0 = tc::smem_desc(sbase + Cf::OFF_M, 16, 1024, tc::kSw128);
        const uint64_t dSS0 = tc::smem_desc(sbase + Cf::OFF_SS, 128 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
        const uint64_t dSU0 = tc::smem_desc(sbase + Cf::OFF_SU, 64 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
        const uint64_t dSU20 = tc::smem_desc(sbase + Cf::OFF_SU2, 64 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);

        const size_t st_base = ((size_t)n * H + h) * 128 * 128 + (size_t)tid * 128 + slab * NS;
        float S[NS];
#pragma unroll
        for (int j = 0; j < NS; j += 4) {
            float4 v4 = a.S0 ? *reinterpret_cast<const float4*>(a.S0 + st_base + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
        }
#pragma unroll
        for (int c = 0; c < NS / 8; ++c) st16(smem + Cf::OFF_SS + tc::swz_off(tid, c, Cf::ROWB), pack8<false>(S + 8 * c));
        float* nw = reinterpret_cast<float*>(smem + Cf::OFF_NW);
        if (GATED && tid < NS) nw[tid] = 1.f + a.norm_w[slab * NS + tid];
        operands_ready(true);

        // M U of chunk ci (slot bb) -> COL_MU[bb]; by thread 0 once M(ci) has landed.  A wait that runs
        // out is flagged and then completed (the copy always lands), so the MMA is always issued
        // and every commit below arrives.
        auto issue_mu = [&](int ci) -> bool {  // thread 0
            const int bb = ci & 1;
            bool w = tc::mbar_wait_bounded(bar_m + bb, (ci >> 1) & 1, a.budget);
            if (!w) {
                raise_error(kErrTimeout);
                tc::mbar_wait_bounded(bar_m + bb, (ci >> 1) & 1, 4000000000ull);
            }
            const uint64_t am0 = desc_add(dM0, bb * 8192), bu0 = desc_add(dSU0, bb * 64 * Cf::ROWB);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // rows 0-63: M U (rows 64-127 read the next tile: unused)
                tc::mma_f16(tmem + Cf::COL_MU + bb * NS, desc_add(am0, kk * 32), desc_add(bu0, kk * 16 * Cf::ROWB),
                            id_mu, kk > 0);
            tc::mma_commit(bar_y);
            if constexpr (!GATED) tc::mma_commit(bar_mfree + bb);  // gated: gate_out frees it
            return w;
        };

        // y of chunk py_x (warps 0-1): y = scale (Gamma_r (Q S) + M U); a full chunk is staged in
        // swizzled rows for one TMA store, a sequence's last partial chunk goes out with plain stores.
        int py_c0 = 0, py_L = 0;
        float py_g = 0.f;         // its Gamma_r (rows 0-63)
        int py_x = -1;            // its index in the sequence (selects TMEM slots, gated buffers, phases)
        bool gated_ok = true;
        // Gated: out = sigmoid(z) y / sqrt(mean_dv(y^2) + eps) (1 + w).  The four slab CTAs of the
        // cluster each hold 32 of the 128 columns of y.  For every chunk each CTA stores every row's
        // partial sum of squares into all four CTAs' shared memory with st.async, whose bytes
        // complete on the receiver's own bar_rs phase (armed by the receiver: 4 x 64 x 4 bytes).
        // y_prev sends and keeps y in yt; gate_out waits for the phase, forms the full mean and gates
        // yt with the z tile the producer loaded beside M.  Every CTA sends and receives exactly
        // nchunks times, also after an error (see the drain below), so no store is still in flight
        // towards a CTA when it exits.
        float yt[NS];
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
        // gated: this row's gate factors sigmoid(z) (1 + w) of chunk py_x -> GZ (row-private, fp32).
        // Waits for the z tile itself (its own acquire of bar_m).
        auto gz_prep = [&]() {
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
        // gated, after send_sums: wait for the cluster's sums of chunk py_x, gate yt, stage it; then the
        // M / z slot is free
        auto gate_out = [&]() {
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
            tc::bar_sync(BID_Y, 64);  // every read of the z slot (gz_prep) is done
            if (tid == 0) tc::mbar_arrive(bar_mfree + bb);
        };
        // y of chunk py_x by warps 0-1, once its M U (issued by thread 0) has completed
        auto y_prev = [&]() -> bool {
            const bool wy = wait_mma(bar_y, ph_y);
            if (tid == 0) tc::bulk_wait_read0();  // YS is free again
            tc::bar_sync(BID_Y, 64);
            if (py_L > 0) {
                const int pb = py_x & 1;
                float t[NS], q1[NS];
                tc::tmem_ld32(trow + Cf::COL_MU + pb * NS, t);
                tc::tmem_ld32(trow + Cf::COL_U + pb * NS, q1);
#pragma unroll
                for (int j = 0; j < NS; ++j) t[j] += py_g * q1[j];
                tc::tmem_ld32(trow + Cf::COL_1B + pb * NS, q1);
#pragma unroll
                for (int j = 0; j < NS; ++j) t[j] = a.scale * (t[j] + py_g * q1[j]);
                if constexpr (GATED) {
                    float ss = 0.f;
#pragma unroll
                    for (int j = 0; j < NS; ++j) {
                        ss += t[j] * t[j];
                        yt[j] = t[j];
                    }
                    send_sums(py_x, ss);
                    gz_prep();
                    gate_out();
                } else {
                    stage_rows(t, a.y_dt);
                }
                tc::fence_async_smem();
                tc::bar_sync(BID_Y, 64);
                if (tid == 0 && py_L == kChunk) {
                    tc::tma_store_3d(&maps.y, slab * NS, h, py_c0, smem + Cf::OFF_YS);
                    tc::bulk_commit();
                }
            }
            return wy && gated_ok;
        };

        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1, kst = c % 3;
            const bool w = tc::mbar_wait_bounded(bar_full + b, (c >> 1) & 1, a.budget);
            if (!(ok = tc::bar_and(BID, 128, w))) {
                if (tid == 0) raise_error(kErrTimeout);
                break;
            }
            tc::tc_fence_after();
            const float* gt = gates(kst);  // Gamma[0:64], f[64:128] of chunk c
            const int c0 = t_begin + c * kChunk, L = min(kChunk, t_end - c0);
            const float gC = gt[63];
            const float gR = tid < 64 ? gt[tid] : 0.f;
            const float fR = tid >= 64 ? gt[tid] : 0.f;

            // [Q; -W] S over dk 0-63 (thread 0) into COL_U[b] and over dk 64-127 (thread 32) into
            // COL_1B[b].  Their sum: Q S in lanes 0-63, -W S in lanes 64-127.  Then thread 0 queues
            // the previous chunk's M U behind it.
            bool wm = true;
            if (tid == 0 || tid == 32) {
                const int hf = tid >> 5;
                const uint64_t a0 = desc_add(dQW0, QWoff(kst) + hf * Cf::QW_HALF);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16(tmem + (hf ? Cf::COL_1B : Cf::COL_U) + b * NS, desc_add(a0, kk * 32),
                                desc_add(dSS0, (hf * 4 + kk) * 16 * Cf::ROWB), id_slab, kk > 0);
                tc::mma_commit(hf ? bar_c2 : bar_c1);
                if (tid == 0 && c > 0) wm = issue_mu(c - 1);
            }
            bool w1 = true, w2 = true, wy = true;
            if (warp >= 2) {
                // U = U~ - W S (fp16, for M U), U' = f U (fp16, for K^T U'), then K^T U' at once
                w1 = wait_mma(bar_c1, ph_c1);
                w2 = wait_mma(bar_c2, ph_c2);
                float d1[NS], d2[NS];
                tc::tmem_ld32(trow + Cf::COL_U + b * NS, d1);
                tc::tmem_ld32(trow + Cf::COL_1B + b * NS, d2);
                const int r = tid - 64;
                float ut[NS];
                const uint8_t* urow = smem + Cf::OFF_UT + kst * 64 * Cf::ROWB + r * Cf::ROWB;
#pragma unroll
                for (int cc = 0; cc < NS / 8; ++cc) {
                    const uint4 u4 = *reinterpret_cast<const uint4*>(urow + 16 * cc);
                    const uint32_t uw[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = unpack2<false>(uw[e]);
                        ut[8 * cc + 2 * e] = f.x + d1[8 * cc + 2 * e] + d2[8 * cc + 2 * e];
                        ut[8 * cc + 2 * e + 1] = f.y + d1[8 * cc + 2 * e + 1] + d2[8 * cc + 2 * e + 1];
                    }
                }
                uint8_t* su = smem + Cf::OFF_SU + b * 64 * Cf::ROWB;
#pragma unroll
                for (int cc = 0; cc < NS / 8; ++cc) {
                    st16(su + tc::swz_off(r, cc, Cf::ROWB), pack8<false>(ut + 8 * cc));
                    float u2[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) u2[e] = fR * ut[8 * cc + e];
                    st16(smem + Cf::OFF_SU2 + tc::swz_off(r, cc, Cf::ROWB), pack8<false>(u2));
                }
                tc::fence_async_smem();
                tc::tc_fence_before();
                tc::bar_sync(BID_U, 64);
                // K^T U' -> state increment; its completion also releases stage kst
                if (tid == 64) {
                    tc::tc_fence_after();
                    const uint64_t ak0 = desc_add(dK0, Koff(kst) - Cf::OFF_KS);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_f16(tmem + Cf::COL_DS, desc_add(ak0, kk * 2048), desc_add(dSU20, kk * 16 * Cf::ROWB),
                                    id_ds, kk > 0);
                    tc::mma_commit(bar_ds);
                    tc::mma_commit(bar_dsd + kst);
                }
            } else if (c > 0) {
                wy = y_prev();  // warps 0-1: y of chunk c - 1 meanwhile
            }
            const bool w3 = wait_mma(bar_ds, ph_ds);
            {
                float t[NS];
                tc::tmem_ld32(trow + Cf::COL_DS, t);
#pragma unroll
                for (int j = 0; j < NS; ++j) S[j] = gC * S[j] + t[j];
#pragma unroll
                for (int cc = 0; cc < NS / 8; ++cc) st16(smem + Cf::OFF_SS + tc::swz_off(tid, cc, Cf::ROWB), pack8<false>(S + 8 * cc));
            }
            py_c0 = c0;
            py_L = L;
            py_g = gR;
            py_x = c;
            if (!(ok = operands_ready(wm && w1 && w2 && wy && w3))) break;
        }
        if (ok && nchunks > 0) {  // the last chunk's M U and y
            bool wm = true;
            if (tid == 0) wm = issue_mu(nchunks - 1);
            bool wy = true;
            if (warp < 2) wy = y_prev();
            ok = tc::bar_and(BID, 128, wm && wy);
        }
        // every MMA of the three issuing threads has completed before TMEM is freed
        if (tid == 0 || tid == 32 || tid == 64) tc::mma_commit(bar_drain);
        tc::mbar_wait_bounded(bar_drain, 0, 4000000000ull);
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
        // Copies and conversions only: every product of the chunk that does not involve the state
        // (-W, U~, M) and its gates come from chunk_ut_kernel's record.  Software-pipelined one
        // chunk ahead of the chain: while the chain works on chunk c, the producer issues the
        // copies of chunk c + 2 into the stage chunk c - 1 has released, and finishes chunk c + 1
        // (waits for its copies, converts bf16 K and Q to fp16, hands it over).
        constexpr int BID = 2;
        const int it = tid - 128;
        tc::wait_prerequisites();  // the records of chunk_ut_kernel are complete and visible
        bool ok = true;

        // copies are issued by one thread of warp 6
        constexpr int kIssuer = 64;
        // copies in flight into this CTA's shared memory, for the exit drain
        int st_issued = -1, st_landed = -1, m_last0 = -1, m_last1 = -1;
        auto rec_ptr = [&](int ci) {
            return reinterpret_cast<const uint8_t*>(a.workspace) + ((size_t)(rec_base + ci) * H + h) * kRecBytes;
        };
        // K of chunk ci -> stage ci % 3; Q of ci -> rows 0-63 of [Q;-W] stage ci % 3; from the record:
        // -W -> rows 64-127, this slab's U~ -> U~ stage, the gates -> gate stage
        auto issue_stage = [&](int ci) {
            st_issued = ci;
            if (it != kIssuer) return;
            const int c0 = t_begin + ci * kChunk, s = ci % 3;
            uint64_t* bk = bar_kv + s;
            tc::mbar_arrive_expect_tx(bk, Cf::K_TX);
            tc::tma_load_3d(smem + Koff(s), &maps.k, 0, h, c0, bk);
            tc::tma_load_3d(smem + Koff(s) + Cf::K_HALF, &maps.k, 64, h, c0, bk);
            uint8_t* qw = smem + QWoff(s);
            const uint8_t* rp = rec_ptr(ci);
            tc::mbar_arrive_expect_tx(bar_q + s, Cf::OP_TX);
            tc::tma_load_3d(qw, &maps.q, 0, h, c0, bar_q + s);
            tc::tma_load_3d(qw + Cf::QW_HALF, &maps.q, 64, h, c0, bar_q + s);
            tc::bulk_g2s(qw + 64 * 128, rp + kRecW, 8192, bar_q + s);
            tc::bulk_g2s(qw + Cf::QW_HALF + 64 * 128, rp + kRecW + 8192, 8192, bar_q + s);
            tc::bulk_g2s(smem + Cf::OFF_UT + s * 64 * Cf::ROWB, rp + kRecU + slab * kRecUSlab, 64 * Cf::ROWB,
                         bar_q + s);
            tc::bulk_g2s(smem + Cf::OFF_GT + s * 512, rp + kRecG, 512, bar_q + s);
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
        // chunk ci landed -> bf16 K and Q to fp16 in place -> handed to the chain (full[ci & 1])
        auto finish = [&](int ci) -> bool {
            const int s = ci % 3;
            bool w = tc::mbar_wait_bounded(bar_kv + s, (ci / 3) & 1, a.budget);
            w = w && tc::mbar_wait_bounded(bar_q + s, (ci / 3) & 1, a.budget);
            if (!tc::bar_and(BID, 128, w)) {
                if (it == 0) raise_error(kErrTimeout);
                return false;
            }
            st_landed = ci;
            if constexpr (BF) {
                // bf16 -> fp16 is exact for |x| >= 2^-14; the smaller entries of a unit-norm key or
                // query lose at most 2^-25 absolute
                to_f16_block<128, 2 * Cf::K_HALF>(smem + Koff(s), it);
                to_f16_block<128, 64 * 128>(smem + QWoff(s), it);               // Q rows of half 0
                to_f16_block<128, 64 * 128>(smem + QWoff(s) + Cf::QW_HALF, it);  // Q rows of half 1
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::bar_sync(BID, 128);
            if (it == 0) tc::mbar_arrive(bar_full + (ci & 1));
            return true;
        };
        if (it == kIssuer) {
            tc::prefetch_tmap(&maps.k);
            tc::prefetch_tmap(&maps.q);
            if constexpr (GATED) tc::prefetch_tmap(&maps.z);
        }
        if (nchunks > 0) issue_stage(0);
        if (nchunks > 1) issue_stage(1);
        if (nchunks > 0) ok = finish(0);

        for (int c = 0; ok && c < nchunks; ++c) {
            // chunk c - 1's state MMA done: stage (c + 2) % 3, which it last read, is free, and the
            // chain has taken chunk c - 1 from full[(c + 1) & 1], so handing over chunk c + 1 there
            // cannot overtake it
            if (c >= 1) {
                const bool w = tc::mbar_wait_bounded(bar_dsd + (c - 1) % 3, ((c - 1) / 3) & 1, a.budget);
                if (!(ok = tc::bar_and(BID, 128, w))) {
                    if (it == 0) raise_error(kErrTimeout);
                    break;
                }
            }
            if (c + 2 < nchunks) issue_stage(c + 2);
            if (c + 1 < nchunks && !(ok = finish(c + 1))) break;
            // M of chunk c, once M U of c - 2 has read the slot (M U of c is issued during chunk c + 1)
            if (it == kIssuer) {
                if (tc::mbar_wait_bounded(bar_mfree + (c & 1), ((c >> 1) & 1) ^ 1, a.budget)) issue_m(c);
                else raise_error(kErrTimeout);
            }
        }
        // never leave with copies into this CTA's shared memory in flight
        for (int ci = max(st_landed + 1, 0); ci <= st_issued; ++ci) {  // at most two outstanding
            tc::mbar_wait_bounded(bar_kv + ci % 3, (ci / 3) & 1, 4000000000ull);
            tc::mbar_wait_bounded(bar_q + ci % 3, (ci / 3) & 1, 4000000000ull);
        }
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
        chunk_ut_kernel<BF><<<(unsigned)(nvc * a.H), UtCfg::THREADS, UtCfg::BYTES, st>>>(a, maps);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const unsigned grid = (unsigned)((long long)a.num_seqs * a.H * (128 / NS));  // <= 2^31 (host check)
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
        !encode_map_3d(&maps.v, a.v, a.in_dt, a.N, a.H, 128, 64, kChunk, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map_3d(&maps.y, gated ? a.out : a.y, st_dt, a.N, a.H, 128, NS, kChunk, yswz) ||
        (gated && !encode_map_3d(&maps.z, a.z, a.z_dt, a.N, a.H, 128, NS, kChunk, CU_TENSOR_MAP_SWIZZLE_64B))) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaSuccess;
    }
    return a.in_dt == kBF16 ? chunk_tc_launch_t<true>(a, maps, st) : chunk_tc_launch_t<false>(a, maps, st);
}

}  // namespace gdn
