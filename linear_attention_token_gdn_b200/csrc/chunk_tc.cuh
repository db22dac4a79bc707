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
//   chunk_ut_kernel     one CTA per (chunk, head), fully parallel, three CTAs per SM, on
//                       warp-level tensor-core products (mma.sync): [K;Q] K^T on the 16-bit
//                       inputs as stored, the decay masks on the accumulators, the
//                       unit-lower-triangular inverse T in fp32, then W = T_w K and U~ = T_u V
//                       with T_w = T diag(beta Gamma) and T_u = T diag(beta) in fp16.  Writes a
//                       40.5 KB record per (chunk, head) by bulk copies: -W and M in the
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
// The chain's operands are 16-bit with fp32 accumulation in TMEM.  A tcgen05.mma instruction
// with M = 128 costs the SM's MMA pipe about 95 cycles for any N up to 64 (N = 128: about 147,
// N = 256: about 173, measured), so its products are shaped to use few instructions, and the
// per-(chunk, head) products are formed once in chunk_ut_kernel rather than once per slab.
// bf16 inputs must lie inside the fp16 range (|x| < 65504), as unit-norm keys and queries do.  [K;Q] K^T reads q and k exactly as stored.  Every product of the
// chain runs on fp16 operands (11 significant bits): bf16 q, k and v are converted to fp16 (exact
// for |x| >= 2^-14; in registers in chunk_ut_kernel, in shared memory when they land in the chain), and their partners T_w, W, S and U'
// are formed in fp16.  bf16 partners (8 bits) would let the error of a row whose y is small
// exceed the bound once eq. (11) normalises that row.  U' = f U enters as one fp16 value (the
// state's error stays near 5e-4 of its scale, well inside the bound).
// Operand tiles use the 128B / 64B swizzled canonical layouts, so one tile serves as K-major
// or MN-major operand.  Every wait is bounded (ChunkArgs::budget clock cycles); a wait that
// runs out sets the device error word, lets in-flight MMAs and copies drain, and the CTA
// returns (after freeing TMEM, in the chain).
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
constexpr int kRecU = 24576;       // U~: four 32-column dv slabs, each [64 rows x 64 B] 64B-swizzled
                                   // (16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3))
constexpr int kRecUSlab = 4096;
constexpr int kRecG = 40960;       // Gamma_r = exp(gamma_r) [64] then f_r = exp(gamma_C - gamma_r) [64], fp32
constexpr int kRecK = 41472;       // K, fp16, two dk halves [64 rows x 128 B] 128B-swizzled K-major
constexpr int kRecQ = 57856;       // Q, fp16, the same layout
constexpr int kRecBytes = 74240;

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

// PREP: the kernel also runs eqs. (6)-(10) (prep fused into the chunked pass): it loads the raw
// projection outputs with the conv history before the chunk, so each tile half holds 72 rows.
template <bool PREP>
struct UtCfgT {
    static constexpr int THREADS = 256;
    // K, Q, V, each two dk (dv) halves of 128-byte rows.  Without PREP: [64 rows x 128 B] as stored
    // (bf16 or fp16), in the 128B-swizzled layout TMA writes.  With PREP: the raw rows of tokens
    // t0 - (W-1) .. t0 + 63, unswizzled, overwritten in place by q, k, v (row r = token t0 + r, the
    // operand format, 128B-swizzled relative to the half's base).  After [K;Q] K^T the Q tile stages
    // M (the record's layout) until it has been stored, then holds [T_w; T_u] (fp16, [128 rows x 128
    // B], same swizzle); -W overwrites K in place in the record's layout (halves 8 KB apart: with
    // 9 KB halves, -W row r of half 1 lands on K row r - 8 of the same columns).
    static constexpr int HS = PREP ? 9216 : 8192;           // bytes per tile half
    static constexpr int OFF_K = 0, OFF_Q = 2 * HS, OFF_V = 4 * HS;
    // fp32 A, turned into T in place [64][LD]; its upper triangle is scratch of the block inverse;
    // once [T_w; T_u] has been formed, it stages U~ (the record's four slabs)
    static constexpr int LD = 68, OFF_A = 6 * HS;
    // per-position vectors (fp32): gamma, beta, beta Gamma, colf [64] each, then rowf [64][4]
    static constexpr int OFF_VEC = OFF_A + 64 * LD * 4;
    static constexpr int V_GAMMA = 0, V_BETA = 64, V_BG = 128, V_COLF = 192, V_ROWF = 256;
    static constexpr int OFF_PSS = OFF_VEC + 4 * (V_ROWF + 256);  // PREP: row sums of squares [q, k][half][64]
    static constexpr int OFF_META = OFF_PSS + (PREP ? 4 * 256 : 0);
    static constexpr int OFF_BAR = OFF_META + 32;           // K and Q landed, V landed
    // the base is aligned to the 1024-byte swizzle atom for TMA's 128B swizzle; the unswizzled raw
    // tiles need 128 bytes (and three CTAs of this size just fit an SM)
    static constexpr int ALIGN = PREP ? 128 : 1024;
    static constexpr int BYTES = OFF_BAR + 16 + ALIGN;
    static_assert(64 * LD * 4 >= 16384 && OFF_A % 1024 == 0, "U~ staging fits over A");
    static_assert(2 * HS >= 16384, "[T_w; T_u] fits in the Q tile");
    static_assert(3 * (BYTES + 1024) <= 228 * 1024, "three CTAs per SM");
};
using UtCfg = UtCfgT<false>;

// Inputs of the fused prep (eqs. (6)-(10)); unused without PREP.
struct PrepIn {
    const float *w_q, *w_k, *w_v;        // conv taps [H*d, W] fp32
    int W;                               // conv width, 1..8
    const void *beta_logit, *alpha_logit;  // [N, H], raw_dt
    const float *A_log, *alpha_bias;     // [H]
    float l2_eps;
    int raw_dt;                          // x_q, x_k, x_v and the logits: bf16 or fp16
};

// Shared-memory byte offset of 16-byte chunk c of row r in a [rows x 128 B] 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void sts32(uint8_t* p, uint32_t v) { *reinterpret_cast<uint32_t*>(p) = v; }

// This lane's two channels (2 lane, 2 lane + 1) of raw row `row` of a 128-byte-row tile half.
__device__ __forceinline__ float2 raw_pair(const uint8_t* half, int row, int lane, int raw_dt) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(half + row * 128 + 4 * lane);
    return raw_dt == kBF16 ? unpack2<true>(w) : unpack2<false>(w);
}

// Eqs. (6)-(8) before the norm: ShortConv -> SiLU of this lane's two channels for the 64 output rows
// of a tile half whose raw row i holds token t0 - (W-1) + i, so output row r (token t0 + r) reads
// raw rows r .. r + W-1, tap j meeting row r + j (the order gdn_prep adds the taps in).  The window
// is right-aligned in eight registers, the taps zero-padded in front, so every index is static.
// first: the chunk starts its sequence, so the W-1 rows before it are the zero history.
// f(r, y0, y1) receives each output row in order; raw row r is not read after output row r.
template <typename F>
__device__ __forceinline__ void conv_silu_half(const uint8_t* half, int W, const float (&wl)[8][2], bool first,
                                               int lane, int raw_dt, F&& f) {
    float2 xw[8];  // at output row r: xw[i] = raw row r + W - 8 + i
#pragma unroll
    for (int i = 1; i < 8; ++i) {
        const int row = W - 8 + i - 1;  // raw row of xw[i] before the first shift
        xw[i] = (row < 0 || (first && row < W - 1)) ? make_float2(0.f, 0.f) : raw_pair(half, row, lane, raw_dt);
    }
#pragma unroll 1
    for (int r0 = 0; r0 < 64; r0 += 4) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = r0 + k;
#pragma unroll
            for (int i = 0; i < 7; ++i) xw[i] = xw[i + 1];
            xw[7] = raw_pair(half, r + W - 1, lane, raw_dt);
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                a0 += wl[i][0] * xw[i].x;
                a1 += wl[i][1] * xw[i].y;
            }
            f(r, __fdividef(a0, 1.0f + __expf(-a0)), __fdividef(a1, 1.0f + __expf(-a1)));
        }
    }
}

// This lane's taps (channels 64 hf + 2 lane, +1 of head h), right-aligned: wl[8 - W + j] = w[c][j].
__device__ __forceinline__ void prep_taps(const float* w, int W, int h, int hf, int lane, float (&wl)[8][2]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int j = i - (8 - W);
#pragma unroll
        for (int u = 0; u < 2; ++u) wl[i][u] = j >= 0 ? w[((size_t)h * 128 + 64 * hf + 2 * lane + u) * W + j] : 0.f;
    }
}

// Output row r of a tile half, in the operand format, over raw row r (its 16-byte chunks swizzled
// relative to the half's base), once every lane of the warp is past reading raw row r.
__device__ __forceinline__ void put_row(uint8_t* half, int r, int lane, uint32_t packed) {
    __syncwarp();
    sts32(half + sw128(r, lane >> 2) + ((lane & 3) << 2), packed);
}

// Virtual chunk v -> (sequence n, chunk j of n) and the bounds [tb, te) of sequence n, from one
// pass over cu_seqlens.  Warp-collective; false if v is past the end.
__device__ bool locate_chunk(const int32_t* cu, int num_seqs, int N, int v, int& n, int& j, int& tb, int& te) {
    const int lane = threadIdx.x & 31;
    int base = 0;
    for (int m0 = 0; m0 < num_seqs; m0 += 32) {
        const int m = m0 + lane;
        int sa = 0, sb = 0;
        if (m < num_seqs) seq_bounds(cu, m, num_seqs, N, sa, sb);
        const int cnt = (sb - sa + kChunk - 1) / kChunk;
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
            tb = __shfl_sync(0xffffffffu, sa, l);
            te = __shfl_sync(0xffffffffu, sb, l);
            return true;
        }
        base += total;
    }
    return false;
}

// Lower 16x8 tile idx (0..19, row-major over 16-row tiles R and 8-column strips j <= 2R + 1).
__device__ __forceinline__ void lower_tile(int idx, int& R, int& j) {
    R = idx < 2 ? 0 : idx < 6 ? 1 : idx < 12 ? 2 : 3;
    j = idx - (R == 0 ? 0 : R == 1 ? 2 : R == 2 ? 6 : 12);
}

// One CTA (eight warps) per (chunk, head), three CTAs per SM, on warp-level tensor-core products
// (mma.sync): each product here is small and triangular, so a tcgen05 round trip (issue, commit,
// TMEM load) would cost more than the arithmetic.
//   1. [K;Q] K^T on the inputs as stored (bf16 or fp16), lower 16x8 tiles only: warp w takes
//      the rows of K (w < 4) or Q (w >= 4) against column strips w % 4 and 7 - w % 4, five tiles.
//   2. The decay masks on the accumulators: A = beta_r exp(gamma_r - gamma_s) (s < r) to fp32
//      shared memory, M = exp(gamma_r - gamma_s) (s <= r) to fp16 and out to the record.
//   3. T = (I + A)^-1 in fp32, in place: 16x16 diagonal blocks by forward substitution, then
//          T21 = -T22 (A21 T11)   for 16x16 blocks, then the same for the 32x32 halves,
//      as mma.sync products of fp32 values split into fp16 pairs (about fp32 accuracy).
//   4. [T_w; T_u] = [T diag(beta Gamma); T diag(beta)] in fp16, then W = T_w K (warps 0-3) and
//      U~ = T_u V (warps 4-7) with K and V converted to fp16 in registers (exact for
//      |x| >= 2^-14), lower blocks only.
//   5. -W, U~ and M leave as bulk copies of tiles staged in the record's layout; the gates
//      Gamma_r and Gamma_C / Gamma_r go to the record directly.
template <bool BF, bool PREP>
__global__ void __launch_bounds__(UtCfg::THREADS, 3) chunk_ut_kernel(const __grid_constant__ ChunkArgs a,
                                                                     const __grid_constant__ ChainMaps maps,
                                                                     const __grid_constant__ PrepIn p) {
    using Cf = UtCfgT<PREP>;
    constexpr int LD = Cf::LD, NT = Cf::THREADS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = PREP ? smem_raw + ((128u - (tc::smem_u32(smem_raw) & 127u)) & 127u) : align_smem_1024(smem_raw);
    const uint32_t sbase = tc::smem_u32(smem);
    float* fA = reinterpret_cast<float*>(smem + Cf::OFF_A);
    float* vb = reinterpret_cast<float*>(smem + Cf::OFF_VEC);
    int* meta = reinterpret_cast<int*>(smem + Cf::OFF_META);
    uint64_t* bar_kq = reinterpret_cast<uint64_t*>(smem + Cf::OFF_BAR);  // K and Q landed
    uint64_t* bar_v = bar_kq + 1;                                        // V landed
    uint8_t* Kt = smem + Cf::OFF_K;
    uint8_t* Qt = smem + Cf::OFF_Q;
    const uint32_t kb = sbase + Cf::OFF_K, qb = sbase + Cf::OFF_Q;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;   // fragment row and column pair of this lane
    const int mi = lane >> 3, rr = lane & 7;   // ldmatrix: the matrix and row this lane addresses
    // heads vary fastest across the grid, so CTAs resident together read whole token rows
    const int H = a.H, v = (int)(blockIdx.x / (unsigned)H), h = (int)(blockIdx.x % (unsigned)H);
    tc::launch_dependents();  // the chain kernel may start its prologue once every CTA is resident

    // ---- locate the chunk; K and Q, then V, as they are stored, by TMA.  Rows past the sequence end
    //      hold other tokens (or the fill of a load past N); they only meet beta = 0 or the
    //      strictly-upper mask, so nothing needs clearing. -------------------------------------------
    if (warp == 0) {
        int n = 0, j = 0, tb = 0, te = 0;
        const bool found = locate_chunk(a.cu, a.num_seqs, a.N, v, n, j, tb, te);
        if (lane == 0) {
            const int t0 = tb + j * kChunk;
            // (bounds-checking build) the record and the chunk's tokens lie inside their tensors;
            // a chunk that fails is skipped before any copy is issued
            const bool use = found && in_bounds(v, chunk_count_bound(a.N, a.num_seqs, a.cu != nullptr)) &&
                             in_bounds(t0, a.N) && in_bounds(te - 1, a.N);
            meta[0] = use;
            meta[1] = t0;
            meta[2] = min(kChunk, te - t0);
            meta[3] = j == 0;
            if (use) {
                // with PREP the maps cover the raw projection outputs, 64 + W - 1 rows from the conv
                // history on (a load before token 0 reads zeros)
                const int row0 = PREP ? t0 - (p.W - 1) : t0;
                const uint32_t half_bytes = PREP ? (64 + p.W - 1) * 128 : 8192;
                tc::mbar_init(bar_kq, 1);
                tc::mbar_init(bar_v, 1);
                tc::fence_mbar_init();
                tc::mbar_arrive_expect_tx(bar_kq, 4 * half_bytes);
                tc::mbar_arrive_expect_tx(bar_v, 2 * half_bytes);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    tc::tma_load_3d(Kt + hf * Cf::HS, &maps.k, 64 * hf, h, row0, bar_kq);
                    tc::tma_load_3d(Qt + hf * Cf::HS, &maps.q, 64 * hf, h, row0, bar_kq);
                }
#pragma unroll
                for (int hf = 0; hf < 2; ++hf)
                    tc::tma_load_3d(smem + Cf::OFF_V + hf * Cf::HS, &maps.v, 64 * hf, h, row0, bar_v);
            }
        }
    }
    __syncthreads();
    if (!meta[0]) return;  // uniform
    const int t0 = meta[1], L = meta[2];
    uint8_t* rec = reinterpret_cast<uint8_t*>(a.workspace) + ((size_t)v * H + h) * kRecBytes;
    const bool first = meta[3] != 0;  // the chunk starts its sequence (PREP: a zero conv history)
    auto drain = [&]() {  // a copy did not land in time: flag it and let every copy finish
        if (tid == 0) {
            raise_error(kErrTimeout);
            tc::mbar_wait_bounded(bar_kq, 0, 4000000000ull);
            tc::mbar_wait_bounded(bar_v, 0, 4000000000ull);
        }
    };

    // ---- gates (warp 1, two positions per lane): gamma = inclusive prefix sum of g inside the
    //      chunk (positions past the sequence end carry g = 0, beta = 0), Gamma = exp(gamma); the
    //      record gets Gamma_r and f_r = exp(gamma_C - gamma_r).  The decay exp(gamma_r - gamma_s)
    //      of a pair in different 16-blocks is split at the end e of s's block into
    //      rowf[r][blk s] = exp(gamma_r - gamma_e) and colf[s] = exp(gamma_e - gamma_s), both <= 1.
    if (warp == (PREP ? 6 : 1)) {
        const int r0 = 2 * lane;
        const size_t i0 = (size_t)(t0 + r0) * H + h;
        float g0 = 0.f, g1 = 0.f, b0 = 0.f, b1 = 0.f;
        if constexpr (PREP) {  // eqs. (9), (10) as gdn_prep forms them
            const float ea = expf(p.A_log[h]), bias = p.alpha_bias[h];
            if (r0 < L) {
                b0 = 1.0f / (1.0f + expf(-ld1(p.beta_logit, p.raw_dt, i0)));
                g0 = -ea * softplusf_(ld1(p.alpha_logit, p.raw_dt, i0) + bias);
            }
            if (r0 + 1 < L) {
                b1 = 1.0f / (1.0f + expf(-ld1(p.beta_logit, p.raw_dt, i0 + H)));
                g1 = -ea * softplusf_(ld1(p.alpha_logit, p.raw_dt, i0 + H) + bias);
            }
        } else {
            g0 = r0 < L ? a.g[i0] : 0.f;
            g1 = r0 + 1 < L ? a.g[i0 + H] : 0.f;
            b0 = r0 < L ? a.beta[i0] : 0.f;
            b1 = r0 + 1 < L ? a.beta[i0 + H] : 0.f;
        }
        float s = g0 + g1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        float ex = __shfl_up_sync(0xffffffffu, s, 1);
        if (lane == 0) ex = 0.f;
        const float gm0 = ex + g0, gm1 = gm0 + g1;
        const float gC = __shfl_sync(0xffffffffu, gm1, 31);
        const float ge = __shfl_sync(0xffffffffu, gm1, lane | 7);  // gamma at the end of this 16-block
        const float G0 = __expf(gm0), G1 = __expf(gm1);
        *reinterpret_cast<float2*>(vb + Cf::V_GAMMA + r0) = make_float2(gm0, gm1);
        *reinterpret_cast<float2*>(vb + Cf::V_BETA + r0) = make_float2(b0, b1);
        *reinterpret_cast<float2*>(vb + Cf::V_BG + r0) = make_float2(b0 * G0, b1 * G1);
        *reinterpret_cast<float2*>(vb + Cf::V_COLF + r0) = make_float2(__expf(ge - gm0), __expf(ge - gm1));
        float rf0[4], rf1[4];
#pragma unroll
        for (int B = 0; B < 4; ++B) {
            const float gb = __shfl_sync(0xffffffffu, gm1, 8 * B + 7);  // gamma at the end of block B
            rf0[B] = B < (r0 >> 4) ? __expf(gm0 - gb) : 0.f;
            rf1[B] = B < (r0 >> 4) ? __expf(gm1 - gb) : 0.f;
        }
        *reinterpret_cast<float4*>(vb + Cf::V_ROWF + 4 * r0) = make_float4(rf0[0], rf0[1], rf0[2], rf0[3]);
        *reinterpret_cast<float4*>(vb + Cf::V_ROWF + 4 * r0 + 4) = make_float4(rf1[0], rf1[1], rf1[2], rf1[3]);
        float* rg = reinterpret_cast<float*>(rec + kRecG);
        *reinterpret_cast<float2*>(rg + r0) = make_float2(G0, G1);
        *reinterpret_cast<float2*>(rg + 64 + r0) = make_float2(__expf(gC - gm0), __expf(gC - gm1));
    }
    if (!__syncthreads_and(tc::mbar_wait_bounded(bar_kq, 0, a.budget))) {
        drain();
        return;
    }
    if constexpr (PREP) {
        // ---- eqs. (6)-(8): q, k, v from the raw rows, in place.  Warps 0-5: tensor w >> 1 (q, k, v),
        //      half w & 1, all 64 rows.  For q and k pass one sums each row's squares over this half
        //      (the L2Norm needs both halves, exchanged through shared memory between the two warps
        //      of the tensor); pass two recomputes the conv, normalises, rounds to the operand format
        //      and writes each row over its raw row.  v: one pass, no norm. ------------------------
        bool okv = true;
        if (warp < 6) {
            const int ten = warp >> 1, hf = warp & 1;
            uint8_t* half = (ten == 0 ? Qt : ten == 1 ? Kt : smem + Cf::OFF_V) + hf * Cf::HS;
            float wl[8][2];
            prep_taps(ten == 0 ? p.w_q : ten == 1 ? p.w_k : p.w_v, p.W, h, hf, lane, wl);
            if (ten < 2) {
                float* pss = reinterpret_cast<float*>(smem + Cf::OFF_PSS) + ten * 128;
                conv_silu_half(half, p.W, wl, first, lane, p.raw_dt, [&](int r, float y0, float y1) {
                    const float ss = warp_sum(y0 * y0 + y1 * y1);
                    if (lane == 0) pss[hf * 64 + r] = ss;
                });
                tc::bar_sync(2 + ten, 64);
                conv_silu_half(half, p.W, wl, first, lane, p.raw_dt, [&](int r, float y0, float y1) {
                    const float inv = rsqrtf(pss[r] + pss[64 + r] + p.l2_eps);
                    put_row(half, r, lane, pack2<BF>(y0 * inv, y1 * inv));
                });
            } else {
                okv = tc::mbar_wait_bounded(bar_v, 0, a.budget);
                if (okv)
                    conv_silu_half(half, p.W, wl, first, lane, p.raw_dt,
                                   [&](int r, float y0, float y1) { put_row(half, r, lane, pack2<BF>(y0, y1)); });
            }
        }
        if (!__syncthreads_and(okv)) {
            drain();
            return;
        }
    }

    // ---- 1-2. [K;Q] K^T and the masks --------------------------------------------------------------
    {
        const int mat = warp >> 2, jj = warp & 3;             // mat 0: A from K rows, 1: M from Q rows
        const int strip[2] = {jj, 7 - jj};                     // 8-column strips of this warp
        const int rmin0 = jj >> 1, rmin1 = (7 - jj) >> 1;      // first 16-row tile at or below the diagonal
        const uint32_t aop = mat ? qb : kb;
        const int brow = 8 * (mi < 2 ? strip[0] : strip[1]) + rr;
        float acc[4][2][4];
#pragma unroll
        for (int R = 0; R < 4; ++R)
#pragma unroll
            for (int si = 0; si < 2; ++si)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[R][si][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t hoff = (kk >> 2) * Cf::HS;
            const int c = 2 * (kk & 3);
            uint32_t bq[4];
            wm::ldsm_x4(kb + hoff + sw128(brow, c + (mi & 1)), bq);
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                if (R < rmin0) continue;  // warp-uniform; rmin0 <= rmin1
                uint32_t af[4];
                wm::ldsm_x4(aop + hoff + sw128(16 * R + rr + 8 * (mi & 1), c + (mi >> 1)), af);
                wm::mma16816x<BF>(acc[R][0], af, bq[0], bq[1]);
                if (R >= rmin1) wm::mma16816x<BF>(acc[R][1], af, bq[2], bq[3]);
            }
        }
        // masks on the accumulators: element e of tile (R, si) is row 16R + g8 + 8 (e >> 1),
        // column 8 strip + 2 t4 + (e & 1); its column block is strip / 2
#pragma unroll
        for (int si = 0; si < 2; ++si) {
            const int s0 = 8 * strip[si] + 2 * t4, rmin = si ? rmin1 : rmin0, sb = strip[si] >> 1;
            const float2 gs = *reinterpret_cast<const float2*>(vb + Cf::V_GAMMA + s0);
            const float2 cf = *reinterpret_cast<const float2*>(vb + Cf::V_COLF + s0);
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                if (R < rmin) continue;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = 16 * R + g8 + 8 * hh;
                    const float sc = mat ? 1.f : vb[Cf::V_BETA + r];
                    float f0, f1;
                    if (sb < R) {  // an earlier block: the split factors (warp-uniform branch)
                        const float rf = vb[Cf::V_ROWF + 4 * r + sb] * sc;
                        f0 = rf * cf.x;
                        f1 = rf * cf.y;
                    } else {       // the row's own block
                        const float gr = vb[Cf::V_GAMMA + r];
                        f0 = (mat ? s0 <= r : s0 < r) ? sc * __expf(gr - gs.x) : 0.f;
                        f1 = (mat ? s0 + 1 <= r : s0 + 1 < r) ? sc * __expf(gr - gs.y) : 0.f;
                    }
                    acc[R][si][2 * hh] *= f0;
                    acc[R][si][2 * hh + 1] *= f1;
                }
            }
        }
        if (mat == 0) {
#pragma unroll
            for (int R = 0; R < 4; ++R)
#pragma unroll
                for (int si = 0; si < 2; ++si)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                        *reinterpret_cast<float2*>(fA + (16 * R + g8 + 8 * hh) * LD + 8 * strip[si] + 2 * t4) =
                            make_float2(acc[R][si][2 * hh], acc[R][si][2 * hh + 1]);
        } else {
            // M straight from the registers to the record (its upper blocks as zeros)
#pragma unroll
            for (int R = 0; R < 4; ++R)
#pragma unroll
                for (int si = 0; si < 2; ++si)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int r = 16 * R + g8 + 8 * hh;
                        *reinterpret_cast<uint32_t*>(rec + kRecM + sw128(r, strip[si]) + 4 * t4) =
                            pack2<false>(acc[R][si][2 * hh], acc[R][si][2 * hh + 1]);
                    }
        }
    }
    __syncthreads();

    // ---- 3. T = (I + A)^-1.  The diagonal blocks (warps 0-3, lane = column), in place once the warp
    //      has read its block ----------------------------------------------------------------------
    if (warp < 4) {
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
                float s0 = 0.f, s1 = 0.f;  // two partial sums shorten the dependent chain
#pragma unroll
                for (int s = 0; s < r; ++s) {
                    if (s & 1) s1 -= arow[s] * xs[s];
                    else s0 -= arow[s] * xs[s];
                }
                xs[r] = ((r == jc) ? 1.f : 0.f) + (s0 + s1);
            }
            __syncwarp(0x0000ffffu);
#pragma unroll
            for (int r = 0; r < 16; ++r) fA[(b0 + r) * LD + b0 + jc] = xs[r];
        }
    } else {
        // meanwhile K and Q in fp16 to the record (the chain's operands), converted in place (exact
        // for |x| >= 2^-14); W = T_w K then reads K as is
        if constexpr (BF) {
            to_f16_block<128, 8192>(Kt, tid - 128);
            to_f16_block<128, 8192>(Kt + Cf::HS, tid - 128);
            to_f16_block<128, 8192>(Qt, tid - 128);
            to_f16_block<128, 8192>(Qt + Cf::HS, tid - 128);
        }
        tc::fence_async_smem();
        tc::bar_sync(1, 128);
        if (tid == 128) {
            tc::bulk_s2g(rec + kRecK, Kt, 8192);
            tc::bulk_s2g(rec + kRecK + 8192, Kt + Cf::HS, 8192);
            tc::bulk_s2g(rec + kRecQ, Qt, 8192);
            tc::bulk_s2g(rec + kRecQ + 8192, Qt + Cf::HS, 8192);
            tc::bulk_commit();
        }
    }
    __syncthreads();
    // T_i,i-1 = -T_ii (A_i,i-1 T_i-1,i-1) for i = 1, 3 (warps 0, 1), over A_i,i-1; the product in
    // brackets goes to the (unused) upper block at rows 0-15, columns 32 + 16 warp
    if (warp < 2) {
        const int bi = 2 * warp + 1, bj = bi - 1;
        float* x1 = fA + 32 + 16 * warp;
        uint32_t ah[4], al[4], bh[2], bl[2];
        wm::load_a(fA, LD, 16 * bi, 16 * bj, 1.f, ah, al);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            wm::load_b(fA, LD, 16 * bj, 16 * bj + 8 * nt, bh, bl);
            wm::mma_split(d, ah, al, bh, bl);
            wm::store_c(x1, LD, 0, 8 * nt, d);
        }
        __syncwarp();
        wm::load_a(fA, LD, 16 * bi, 16 * bi, -1.f, ah, al);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float e[4] = {0.f, 0.f, 0.f, 0.f};
            wm::load_b(x1, LD, 0, 8 * nt, bh, bl);
            wm::mma_split(e, ah, al, bh, bl);
            wm::store_c(fA, LD, 16 * bi, 16 * bj + 8 * nt, e);
        }
    }
    __syncthreads();
    // X = A[32:64, 0:32] T[0:32, 0:32] into the upper block rows 0-31, columns 32-63; then
    // T[32:64, 0:32] = -T[32:64, 32:64] X over A, one 16x8 tile per warp, skipping the zero
    // upper-right 16x16 blocks
    {
        const int mt = warp >> 2, nt = warp & 3;
        float* x2 = fA + 32;
        uint32_t ah[4], al[4], bh[2], bl[2];
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            if (kt == 0 && nt >= 2) continue;  // T[0:16, 16:32] = 0
            wm::load_a(fA, LD, 32 + 16 * mt, 16 * kt, 1.f, ah, al);
            wm::load_b(fA, LD, 16 * kt, 8 * nt, bh, bl);
            wm::mma_split(d, ah, al, bh, bl);
        }
        wm::store_c(x2, LD, 16 * mt, 8 * nt, d);
        if (tid == 128) tc::bulk_wait_read0();  // Q and K have left their tiles ([T_w; T_u], -W overwrite them)
        __syncthreads();
        float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            if (mt == 0 && kt == 1) continue;  // T[32:48, 48:64] = 0
            wm::load_a(fA, LD, 32 + 16 * mt, 32 + 16 * kt, -1.f, ah, al);
            wm::load_b(x2, LD, 16 * kt, 8 * nt, bh, bl);
            wm::mma_split(e, ah, al, bh, bl);
        }
        wm::store_c(fA, LD, 32 + 16 * mt, 8 * nt, e);
    }
    __syncthreads();

    // ---- 4. [T_w; T_u] (fp16, rows 0-63 and 64-127 of the Q tile), lower triangle incl. diagonal --
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int idx = tid + NT * q, which = idx >> 9, r = (idx >> 3) & 63, cc = idx & 7;
        const float4 t0v = lds4(fA + r * LD + 8 * cc), t1v = lds4(fA + r * LD + 8 * cc + 4);
        const float* sv = vb + (which ? Cf::V_BETA : Cf::V_BG) + 8 * cc;  // column scales beta Gamma, beta
        const float4 b0v = lds4(sv), b1v = lds4(sv + 4);
        float t8[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
        const float s8[8] = {b0v.x, b0v.y, b0v.z, b0v.w, b1v.x, b1v.y, b1v.z, b1v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) t8[e] = (8 * cc + e <= r) ? t8[e] * s8[e] : 0.f;
        st16(Qt + sw128(64 * which + r, cc), pack8<false>(t8));
    }
    const bool isU = warp >= 4;
    if (!__syncthreads_and(isU && !PREP ? tc::mbar_wait_bounded(bar_v, 0, a.budget) : true)) {
        if (tid == 128) tc::bulk_wait0();
        drain();
        return;
    }

    // W = T_w K (warps 0-3) and U~ = T_u V (warps 4-7), 32 output columns per warp in two passes
    // of 16; row tile R of the triangular T needs k-steps 0..R only.  -W overwrites the K columns
    // this warp alone has read (the record's dk-half layout); U~ goes over A, which nothing reads
    // any more (the record's 64B-swizzled 32-column slabs).
    {
        const uint32_t bopnd = isU ? sbase + Cf::OFF_V : kb;
        const uint32_t aopnd = qb + (isU ? 64 * 128 : 0);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int n0 = 32 * (warp & 3) + 16 * p, hf = n0 >> 6, cb = (n0 & 63) >> 3;
            float acc[4][2][4];
#pragma unroll
            for (int R = 0; R < 4; ++R)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[R][nt][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t bv[4];
                wm::ldsm_x4_t(bopnd + hf * Cf::HS + sw128(16 * kk + rr + 8 * (mi & 1), cb + (mi >> 1)), bv);
                if (BF && isU) {  // V as stored; K is fp16 by now
#pragma unroll
                    for (int e = 0; e < 4; ++e) bv[e] = wm::bf2_to_h2(bv[e]);
                }
#pragma unroll
                for (int R = kk; R < 4; ++R) {
                    uint32_t af[4];
                    wm::ldsm_x4(aopnd + sw128(16 * R + rr + 8 * (mi & 1), 2 * kk + (mi >> 1)), af);
                    wm::mma16816x<false>(acc[R][0], af, bv[0], bv[1]);
                    wm::mma16816x<false>(acc[R][1], af, bv[2], bv[3]);
                }
            }
            if (!isU) __syncwarp();  // every lane has read these K columns
#pragma unroll
            for (int R = 0; R < 4; ++R)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int r = 16 * R + g8 + 8 * hh;
                        const float x0 = acc[R][nt][2 * hh], x1 = acc[R][nt][2 * hh + 1];
                        if (!isU) {
                            sts32(Kt + hf * 8192 + sw128(r, cb + nt) + 4 * t4, pack2<false>(-x0, -x1));
                        } else {
                            const int n = n0 + 8 * nt + 2 * t4;
                            sts32(smem + Cf::OFF_A + (n >> 5) * kRecUSlab + tc::swz_off(r, (n & 31) >> 3, 64) +
                                      (n & 7) * 2,
                                  pack2<false>(x0, x1));
                        }
                    }
        }
    }
    tc::fence_async_smem();
    __syncthreads();
    if (tid == 0) {
        tc::bulk_s2g(rec + kRecW, Kt, 16384);
        tc::bulk_s2g(rec + kRecU, smem + Cf::OFF_A, 16384);
        tc::bulk_commit();
    }
    // the CTA may leave once its staged tiles have been read; the writes complete before any later
    // grid (or programmatic dependent waiting on this one) reads them
    if (tid == 0 || tid == 128) tc::bulk_wait_read0();
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
    static constexpr int OFF_UT = OFF_KS + 3 * 2 * K_HALF;     // [3 stages] U~ slab fp16 [64 x ROWB], 64B-swizzled
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
            } else if (tid < py_L && in_bounds(py_c0 + tid, a.N)) {
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
                const uint8_t* ust = smem + Cf::OFF_UT + kst * 64 * Cf::ROWB;
#pragma unroll
                for (int cc = 0; cc < NS / 8; ++cc) {
                    const uint4 u4 = *reinterpret_cast<const uint4*>(ust + tc::swz_off(r, cc, 64));
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
        // Everything of chunk ci from its record, already fp16 in the operand layouts: K -> stage
        // ci % 3; Q -> rows 0-63 and -W -> rows 64-127 of [Q;-W] stage ci % 3; this slab's U~ -> U~
        // stage; the gates -> gate stage
        auto issue_stage = [&](int ci) {
            st_issued = ci;
            if (it != kIssuer) return;
            const int s = ci % 3;
            uint64_t* bk = bar_kv + s;
            const uint8_t* rp = rec_ptr(ci);
            tc::mbar_arrive_expect_tx(bk, Cf::K_TX);
            tc::bulk_g2s(smem + Koff(s), rp + kRecK, 8192, bk);
            tc::bulk_g2s(smem + Koff(s) + Cf::K_HALF, rp + kRecK + 8192, 8192, bk);
            uint8_t* qw = smem + QWoff(s);
            tc::mbar_arrive_expect_tx(bar_q + s, Cf::OP_TX);
            tc::bulk_g2s(qw, rp + kRecQ, 8192, bar_q + s);
            tc::bulk_g2s(qw + Cf::QW_HALF, rp + kRecQ + 8192, 8192, bar_q + s);
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
        // chunk ci landed -> handed to the chain (full[ci & 1])
        auto finish = [&](int ci) -> bool {
            const int s = ci % 3;
            bool w = tc::mbar_wait_bounded(bar_kv + s, (ci / 3) & 1, a.budget);
            w = w && tc::mbar_wait_bounded(bar_q + s, (ci / 3) & 1, a.budget);
            if (!tc::bar_and(BID, 128, w)) {
                if (it == 0) raise_error(kErrTimeout);
                return false;
            }
            st_landed = ci;
            tc::tc_fence_before();
            tc::bar_sync(BID, 128);
            if (it == 0) tc::mbar_arrive(bar_full + (ci & 1));
            return true;
        };
        if (it == kIssuer && GATED) tc::prefetch_tmap(&maps.z);
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

// ut_maps: the tiles chunk_ut_kernel loads (q, k, v, or with PREP the raw projection outputs);
// maps: the chain's (k and q as the chain reads them, y or out, z).
template <bool BF, bool PREP>
inline cudaError_t chunk_tc_launch_t(const ChunkArgs& a, const ChainMaps& ut_maps, const ChainMaps& maps, const PrepIn& p,
                                     cudaStream_t st) {
    constexpr int NS = 32;
    using Ch = ChainCfg<NS>;
    using Ut = UtCfgT<PREP>;
    cudaError_t e = cudaFuncSetAttribute(chunk_ut_kernel<BF, PREP>, cudaFuncAttributeMaxDynamicSharedMemorySize, Ut::BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_chain_kernel<NS, BF, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, Ch::BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_chain_kernel<NS, BF, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, Ch::BYTES);
    if (e != cudaSuccess) return e;
    const long long nvc = chunk_count_bound(a.N, a.num_seqs, a.cu != nullptr);
    if (nvc > 0) {
        LaunchScope timed(st, PREP ? "chunk_ut_prep_kernel" : "chunk_ut_kernel");
        chunk_ut_kernel<BF, PREP><<<(unsigned)(nvc * a.H), Ut::THREADS, Ut::BYTES, st>>>(a, ut_maps, p);
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
    const PrepIn none = {};
    return a.in_dt == kBF16 ? chunk_tc_launch_t<true, false>(a, maps, maps, none, st)
                            : chunk_tc_launch_t<false, false>(a, maps, maps, none, st);
}

// The chunked path with eqs. (6)-(10) fused into chunk_ut_kernel: x_q, x_k, x_v (p.raw_dt) are
// the projection outputs; a.in_dt is the operand format q, k, v are rounded to (bf16 or fp16).
// a.q, a.k, a.v, a.g, a.beta are unused.
inline cudaError_t chunk_tc_prep_launch(const ChunkArgs& a, const PrepIn& p, const void* x_q, const void* x_k,
                                        const void* x_v, cudaStream_t st, const char** why) {
    *why = nullptr;
    if (a.chunk != kChunk) {
        *why = "only chunk = 64 is built";
        return cudaSuccess;
    }
    constexpr int NS = 32;
    const CUtensorMapSwizzle yswz = a.y_dt == kF32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    ChainMaps raw = {}, maps = {};  // the chain reads K and Q from the records
    const uint32_t rows = 64 + p.W - 1;
    if (!encode_map_3d(&raw.k, x_k, p.raw_dt, a.N, a.H, 128, 64, rows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_map_3d(&raw.q, x_q, p.raw_dt, a.N, a.H, 128, 64, rows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_map_3d(&raw.v, x_v, p.raw_dt, a.N, a.H, 128, 64, rows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_map_3d(&maps.y, a.y, a.y_dt, a.N, a.H, 128, NS, kChunk, yswz)) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaSuccess;
    }
    return a.in_dt == kBF16 ? chunk_tc_launch_t<true, true>(a, raw, maps, p, st)
                            : chunk_tc_launch_t<false, true>(a, raw, maps, p, st);
}

}  // namespace gdn
