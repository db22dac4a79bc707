// chunk_tc.cuh -- chunkwise-parallel GDN prefill on the sm_100a tensor cores.
//
// The recurrence is eqs. (1)-(4) of "On the design of Qwen3.8-Next architecture", section
// 2.1.1.  Unrolling eqs. (1)-(3) over a chunk of C tokens that starts from state S (the
// closed form eq. (5) applied C times), with gamma_r the inclusive prefix sum of
// g = log alpha inside the chunk and Gamma_r = exp(gamma_r), gives
//     A[r,s] = beta_r exp(gamma_r - gamma_s) k_r.k_s   (s < r),   T = (I + A)^-1
//     W  = T diag(beta Gamma) K,      U~ = T diag(beta) V,      U = U~ - W S
//     M[r,s] = exp(gamma_r - gamma_s) q_r.k_s           (s <= r)
//     Y  = diag(Gamma) Q S + M U,     S' = Gamma_C S + (diag(Gamma_C / Gamma) K)^T U
// Every decay factor is exp(<= 0): masks are applied elementwise to the fp32 products in
// the TMEM epilogue, never factored as Gamma_r / Gamma_s.  For s in an earlier 16-row
// block than r the factor is split at the end e of s's block,
//     exp(gamma_r - gamma_s) = exp(gamma_r - gamma_e) * exp(gamma_e - gamma_s),
// both factors <= 1, so a row needs 4 + 16 exponentials instead of 64.
//
// Work decomposition.  The dv columns of S evolve independently (W and A do not depend
// on V), so one CTA owns one (sequence, head, dv-slab of NS columns) and walks the
// sequence chunk by chunk.  Its 256 threads form two warpgroups:
//   * the intra group (warps 4-7) computes everything that does not depend on the state
//     for chunk c+1 -- fp16 operand tiles, masks, the UT transform T, W and U~ -- into one
//     of two shared-memory / TMEM slots, while its loads for chunk c+2 are in flight;
//   * the chain group (warps 0-3) carries the fp32 state (one row per thread, in
//     registers) through chunk c with two dependent tensor-core round trips:
//         [W;Q] S                         -> U = U~ - W S (fp16 operand), Q S kept
//         [T_w;M] U  and  Kg^T U          -> Y = Gamma (Q S) + M U,  S' = Gamma_C S + Kg^T U
// Slots are handed over with mbarriers (full: intra -> chain, empty: chain -> intra).
// Products on tcgen05 (fp16 operands, fp32 accumulation in TMEM):
//     [K;Q] K^T            (M=128, N=64,  K=128)   -> A (rows 0-63) and M (rows 64-127)
//     [T_u;T_w] V_slab     (M=128, N=NS,  K=64)    -> U~ (rows 0-63)
//     [T_u;T_w] K          (M=128, N=128, K=64)    -> W  (rows 64-127)
//     [W;Q] S              (M=128, N=NS,  K=128)   -> W S (rows 0-63), Q S (rows 64-127)
//     [T_w;M] U            (M=128, N=NS,  K=64)    -> M U (rows 64-127)
//     (diag(Gamma_C/Gamma)K)^T U (M=128, N=NS, K=64) -> state increment
// with T_u = T diag(beta), T_w = T diag(beta Gamma).  The 64x64 unit-lower-triangular
// inverse T is formed in fp32 on the CUDA cores (16x16 diagonal blocks by forward
// substitution, then the off-diagonal blocks in three dependent rounds).
// Operand tiles use the 128B (or 64B) swizzled canonical layouts, so one tile (K, or a
// slab tile) serves both as a K-major and as an MN-major operand.
//
// Every wait is bounded (ChunkArgs::budget clock cycles); a wait that runs out sets the
// device error word, lets in-flight MMAs drain, and the CTA returns after freeing TMEM.
#pragma once
#include "common.cuh"
#include "tc_ptx.cuh"

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
};

inline size_t chunk_tc_workspace_bytes(int, int, int, int, int, int) { return 0; }

template <int NS>
struct TcCfg {
    static constexpr int C = 64;
    static constexpr int ROWB = NS * 2;  // bytes per row of a slab tile
    static constexpr uint32_t SWZ = NS == 32 ? tc::kSw64 : tc::kSw128;
    // shared memory (byte offsets from a 1024-aligned base); [2] = per chunk-parity slot
    static constexpr int OFF_X = 0;                          // [2] [K->W ; Q]: 2 x [128 x 128 B]
    static constexpr int OFF_TM = OFF_X + 2 * 32768;         // [2] [T_u; T_w; M]: [192 x 128 B]
    static constexpr int OFF_KG = OFF_TM + 2 * 24576;        // [2] Kg: 2 x [64 x 128 B]
    static constexpr int OFF_VS = OFF_KG + 2 * 16384;        // V slab [64 x ROWB]
    static constexpr int OFF_SS = OFF_VS + 64 * ROWB;        // S operand [128 x ROWB]
    static constexpr int OFF_SU = OFF_SS + 128 * ROWB;       // U operand [64 x ROWB]
    static constexpr int OFF_A = OFF_SU + 64 * ROWB;         // fp32 A [64][65]
    static constexpr int OFF_TF = OFF_A + 64 * 65 * 4;       // fp32 T [64][65]
    static constexpr int OFF_Z = OFF_TF + 64 * 65 * 4;       // fp32 scratch [3][16][17]
    static constexpr int OFF_VEC = OFF_Z + 3 * 16 * 17 * 4;  // [2] gamma, Gamma, beta, colf: 4 x 64 floats
    static constexpr int OFF_META = OFF_VEC + 2 * 1024;      // [2] {c0, L}
    static constexpr int OFF_BAR = OFF_META + 64;            // mbarriers + TMEM base
    static constexpr int BYTES = OFF_BAR + 128 + 1024;       // + alignment slack
    // TMEM columns (fp32 accumulators, lane = output row)
    static constexpr uint32_t COL_QK = 0;
    static constexpr uint32_t COL_UT = 64;                   // [2] x NS
    static constexpr uint32_t COL_W = 64 + 2 * NS;           // 128
    static constexpr uint32_t COL_1 = COL_W + 128;           // NS
    static constexpr uint32_t COL_MU = COL_1 + NS;           // NS
    static constexpr uint32_t COL_DS = COL_MU + NS;          // NS
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(COL_DS + NS <= TMEM_COLS, "TMEM budget");
    static_assert(BYTES <= 232448, "shared memory budget");
};

// 8 consecutive 16-bit input elements -> 8 fp16 values packed in a uint4.
__device__ __forceinline__ uint4 to_f16x8(uint4 u, int in_dt) {
    if (in_dt == kF16) return u;
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w[i]));
        __half2 hv = __floats2half2_rn(f.x, f.y);
        w[i] = *reinterpret_cast<uint32_t*>(&hv);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 pack_f16x8(const float* x) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 hv = __floats2half2_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&hv);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void unpack_f16x8(uint4 u, float* x) {
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __half22float2(*reinterpret_cast<__half2*>(&w[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ uint4 ldg16(const void* p, size_t elem_off) {
    return __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p) + elem_off));
}

template <int NS>
__global__ void __launch_bounds__(256, 1) chunk_fwd_tc_kernel(const __grid_constant__ ChunkArgs a) {
    using Cf = TcCfg<NS>;
    constexpr int C = Cf::C;
    constexpr int NSLAB = 128 / NS;
    constexpr int VU = (64 * NS / 8) / 128;  // 16-byte V pieces per intra thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = tc::smem_u32(smem);
    float* fA = reinterpret_cast<float*>(smem + Cf::OFF_A);
    float* fT = reinterpret_cast<float*>(smem + Cf::OFF_TF);
    float* fZ = reinterpret_cast<float*>(smem + Cf::OFF_Z);
    int* meta = reinterpret_cast<int*>(smem + Cf::OFF_META);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::OFF_BAR);
    uint64_t* bar_i = bars + 0;      // intra-issued MMAs complete
    uint64_t* bar_c = bars + 1;      // chain-issued MMAs complete
    uint64_t* bar_full = bars + 2;   // [2] slot filled by the intra group
    uint64_t* bar_empty = bars + 4;  // [2] slot released by the chain group
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::OFF_BAR + 64);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slab = blockIdx.x % NSLAB;
    const int h = (blockIdx.x / NSLAB) % a.H;
    const int n = blockIdx.x / (NSLAB * a.H);
    const int H = a.H;
    int t_begin, t_end;
    seq_bounds(a.cu, n, a.num_seqs, a.N, t_begin, t_end);
    const int nchunks = (t_end - t_begin + C - 1) / C;

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) tc::mbar_init(bars + i, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, Cf::TMEM_COLS);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's TMEM lanes

    auto vec = [&](int b) { return reinterpret_cast<float*>(smem + Cf::OFF_VEC + b * 1024); };
    auto Xoff = [&](int b) { return Cf::OFF_X + b * 32768; };
    auto TMoff = [&](int b) { return Cf::OFF_TM + b * 24576; };
    auto KGoff = [&](int b) { return Cf::OFF_KG + b * 16384; };

    if (warp < 4) {
        // =============================== chain group ===================================
        constexpr int BID = 1;
        uint32_t ph = 0;
        bool ok = true;
        auto commit_wait = [&]() -> bool {
            if (tid == 0) tc::mma_commit(bar_c);
            bool w = tc::bar_and(BID, 128, tc::mbar_wait_bounded(bar_c, ph, a.budget));
            if (!w) {
                if (tid == 0) raise_error(kErrTimeout);
                tc::mbar_wait_bounded(bar_c, ph, 4000000000ull);
            }
            ph ^= 1u;
            tc::tc_fence_after();
            return w;
        };
        auto operands_ready = [&]() {
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::bar_sync(BID, 128);
            tc::tc_fence_after();
        };
        const uint32_t id_slab = tc::idesc_f16(128, NS, false, true);
        const uint32_t id_ds = tc::idesc_f16(128, NS, true, true);
        const uint32_t sSS = sbase + Cf::OFF_SS, sSU = sbase + Cf::OFF_SU;

        const size_t st_base = ((size_t)n * H + h) * 128 * 128 + (size_t)tid * 128 + slab * NS;
        float S[NS];
#pragma unroll
        for (int j = 0; j < NS; j += 4) {
            float4 v4 = a.S0 ? *reinterpret_cast<const float4*>(a.S0 + st_base + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
        }
#pragma unroll
        for (int c = 0; c < NS / 8; ++c)
            *reinterpret_cast<uint4*>(smem + Cf::OFF_SS + tc::swz_off(tid, c, Cf::ROWB)) = pack_f16x8(S + 8 * c);
        operands_ready();

        float keep[NS];  // rows 64-127: (Q S) row
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (!(ok = tc::bar_and(BID, 128, tc::mbar_wait_bounded(bar_full + b, (c >> 1) & 1, a.budget)))) {
                if (tid == 0) raise_error(kErrTimeout);
                break;
            }
            tc::tc_fence_after();
            const float* vb = vec(b);
            const int c0 = meta[2 * b], L = meta[2 * b + 1];
            const float gC = vb[64 + 63];
            const float gR = tid >= 64 ? vb[64 + tid - 64] : 0.f;
            const uint32_t sX = sbase + Xoff(b), sTM = sbase + TMoff(b), sKG = sbase + KGoff(b);

            // [W;Q] S
            if (tid == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t aw = tc::smem_desc(sX + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, tc::kSw128);
                    const uint64_t bs = tc::smem_desc(sSS + kk * 16 * Cf::ROWB, 128 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
                    tc::mma_f16(tmem + Cf::COL_1, aw, bs, id_slab, kk > 0);
                }
            }
            if (!(ok = commit_wait())) break;

            // U = U~ - W S (rows 0-63) ; Q S kept (rows 64-127)
            {
                float d1[NS];
#pragma unroll
                for (int q4 = 0; q4 < NS / 32; ++q4) tc::tmem_ld32(trow + Cf::COL_1 + 32 * q4, d1 + 32 * q4);
                if (warp < 2) {
                    float ut[NS];
#pragma unroll
                    for (int q4 = 0; q4 < NS / 32; ++q4)
                        tc::tmem_ld32(trow + Cf::COL_UT + b * NS + 32 * q4, ut + 32 * q4);
#pragma unroll
                    for (int j = 0; j < NS; ++j) ut[j] -= d1[j];
#pragma unroll
                    for (int cc = 0; cc < NS / 8; ++cc)
                        *reinterpret_cast<uint4*>(smem + Cf::OFF_SU + tc::swz_off(tid, cc, Cf::ROWB)) =
                            pack_f16x8(ut + 8 * cc);
                } else {
#pragma unroll
                    for (int j = 0; j < NS; ++j) keep[j] = d1[j];
                }
            }
            operands_ready();

            // M U (rows 64-127) and Kg^T U
            if (tid == 0) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bu = tc::smem_desc(sSU + kk * 16 * Cf::ROWB, 64 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
                    const uint64_t am = tc::smem_desc(sTM + 64 * 128 + kk * 32, 16, 1024, tc::kSw128);
                    tc::mma_f16(tmem + Cf::COL_MU, am, bu, id_slab, kk > 0);
                    const uint64_t ak = tc::smem_desc(sKG + kk * 2048, 8192, 1024, tc::kSw128);
                    tc::mma_f16(tmem + Cf::COL_DS, ak, bu, id_ds, kk > 0);
                }
            }
            if (!(ok = commit_wait())) break;
            if (tid == 0) tc::mbar_arrive(bar_empty + b);  // slot b (smem and U~ columns) is free

            {
                float t[NS];
                if (warp >= 2) {
                    const int r = tid - 64;
#pragma unroll
                    for (int q4 = 0; q4 < NS / 32; ++q4) tc::tmem_ld32(trow + Cf::COL_MU + 32 * q4, t + 32 * q4);
                    if (r < L) {
                        const size_t yoff = ((size_t)(c0 + r) * H + h) * 128 + slab * NS;
#pragma unroll
                        for (int j = 0; j < NS; j += 4)
                            st4(a.y, a.y_dt, yoff + j,
                                make_float4(a.scale * (gR * keep[j] + t[j]), a.scale * (gR * keep[j + 1] + t[j + 1]),
                                            a.scale * (gR * keep[j + 2] + t[j + 2]),
                                            a.scale * (gR * keep[j + 3] + t[j + 3])));
                    }
                }
#pragma unroll
                for (int q4 = 0; q4 < NS / 32; ++q4) tc::tmem_ld32(trow + Cf::COL_DS + 32 * q4, t + 32 * q4);
#pragma unroll
                for (int j = 0; j < NS; ++j) S[j] = gC * S[j] + t[j];
#pragma unroll
                for (int cc = 0; cc < NS / 8; ++cc)
                    *reinterpret_cast<uint4*>(smem + Cf::OFF_SS + tc::swz_off(tid, cc, Cf::ROWB)) = pack_f16x8(S + 8 * cc);
            }
            operands_ready();
        }
        if (ok && a.S_T) {
#pragma unroll
            for (int j = 0; j < NS; j += 4)
                *reinterpret_cast<float4*>(a.S_T + st_base + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    } else {
        // =============================== intra group ===================================
        constexpr int BID = 2;
        const int it = tid - 128;
        uint32_t ph = 0;
        bool ok = true;
        auto commit_wait = [&]() -> bool {
            if (it == 0) tc::mma_commit(bar_i);
            bool w = tc::bar_and(BID, 128, tc::mbar_wait_bounded(bar_i, ph, a.budget));
            if (!w) {
                if (it == 0) raise_error(kErrTimeout);
                tc::mbar_wait_bounded(bar_i, ph, 4000000000ull);
            }
            ph ^= 1u;
            tc::tc_fence_after();
            return w;
        };
        auto operands_ready = [&]() {
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::bar_sync(BID, 128);
            tc::tc_fence_after();
        };
        const uint32_t id_qk = tc::idesc_f16(128, 64, false, false);
        const uint32_t id_slab = tc::idesc_f16(128, NS, false, true);
        const uint32_t id_w = tc::idesc_f16(128, 128, false, true);
        const uint32_t sVS = sbase + Cf::OFF_VS;

        // register prefetch of one chunk's inputs (issued a chunk ahead of use)
        uint4 pk[8], pq[8], pv[VU];
        float pg = 0.f, pb = 0.f;
        auto prefetch = [&](int ci) {
            const int c0 = t_begin + ci * C, L = min(C, t_end - c0);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int idx = it + 128 * u, r = idx >> 4, cc = idx & 15;
                const size_t off = ((size_t)(c0 + r) * H + h) * 128 + cc * 8;
                pk[u] = r < L ? ldg16(a.k, off) : make_uint4(0, 0, 0, 0);
                pq[u] = r < L ? ldg16(a.q, off) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < VU; ++u) {
                const int idx = it + 128 * u, r = idx / (NS / 8), cc = idx % (NS / 8);
                pv[u] = r < L ? ldg16(a.v, ((size_t)(c0 + r) * H + h) * 128 + slab * NS + cc * 8) : make_uint4(0, 0, 0, 0);
            }
            if (it < 64) {
                pg = it < L ? a.g[(size_t)(c0 + it) * H + h] : 0.f;
                pb = it < L ? a.beta[(size_t)(c0 + it) * H + h] : 0.f;
            }
        };
        if (nchunks > 0) prefetch(0);

        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const int c0 = t_begin + c * C, L = min(C, t_end - c0);
            float* vb = vec(b);  // gamma[0:64] Gamma[64:128] beta[128:192] colf[192:256]
            const uint32_t sX = sbase + Xoff(b), sTM = sbase + TMoff(b);
            // the chain group must be done with this slot (chunk c-2)
            if (!(ok = tc::bar_and(BID, 128, tc::mbar_wait_bounded(bar_empty + b, ((c >> 1) & 1) ^ 1, a.budget)))) {
                if (it == 0) raise_error(kErrTimeout);
                break;
            }
            tc::tc_fence_after();

            // ---- operand tiles from the prefetched registers; gates ------------------------
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int idx = it + 128 * u, r = idx >> 4, cc = idx & 15, hf = cc >> 3, c8 = cc & 7;
                *reinterpret_cast<uint4*>(smem + Xoff(b) + hf * 16384 + tc::swz_off(r, c8, 128)) = to_f16x8(pk[u], a.in_dt);
                *reinterpret_cast<uint4*>(smem + Xoff(b) + hf * 16384 + tc::swz_off(r + 64, c8, 128)) = to_f16x8(pq[u], a.in_dt);
            }
#pragma unroll
            for (int u = 0; u < VU; ++u) {
                const int idx = it + 128 * u, r = idx / (NS / 8), cc = idx % (NS / 8);
                *reinterpret_cast<uint4*>(smem + Cf::OFF_VS + tc::swz_off(r, cc, Cf::ROWB)) = to_f16x8(pv[u], a.in_dt);
            }
            if (it < 64) {
                float gv = pg;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, gv, o);
                    if (lane >= o) gv += y;
                }
                vb[it] = gv;
                vb[128 + it] = pb;
            }
            if (it == 0) {
                meta[2 * b] = c0;
                meta[2 * b + 1] = L;
            }
            if (c + 1 < nchunks) prefetch(c + 1);  // next chunk's loads overlap this chunk's work
            tc::bar_sync(BID, 128);
            if (it >= 32 && it < 64) vb[it] += vb[31];
            tc::bar_sync(BID, 128);
            if (it < 64) {
                vb[64 + it] = expf(vb[it]);
                vb[192 + it] = expf(vb[(it | 15)] - vb[it]);  // exp(gamma_e - gamma_s), e = end of s's block
            }
            operands_ready();

            // ---- [K;Q] K^T -------------------------------------------------------------------
            if (it == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t d = tc::smem_desc(sX + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, tc::kSw128);
                    tc::mma_f16(tmem + Cf::COL_QK, d, d, id_qk, kk > 0);
                }
            }
            if (!(ok = commit_wait())) break;

            // ---- masks: A (fp32) for the solve, M (fp16 operand); Kg -----------------------------
            {
                float x[64];
                tc::tmem_ld32(trow + Cf::COL_QK, x);
                tc::tmem_ld32(trow + Cf::COL_QK + 32, x + 32);
                const int r = it & 63, R = r >> 4, rl = r & 15;
                const float gr = vb[r];
                const bool isA = it < 64;
                float rowf[4], dg[16];
#pragma unroll
                for (int S = 0; S < 4; ++S) rowf[S] = S < R ? expf(gr - vb[16 * S + 15]) : 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    dg[j] = (isA ? j < rl : j <= rl) ? expf(gr - vb[16 * R + j]) : 0.f;
                const float* colf = vb + 192;
                if (isA) {
                    const float br = vb[128 + r];
#pragma unroll
                    for (int s = 0; s < 64; ++s) {
                        const int S = s >> 4;
                        const float f = S < R ? rowf[S] * colf[s] : (S == R ? dg[s & 15] : 0.f);
                        fA[r * 65 + s] = br * f * x[s];
                    }
                } else {
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        float m[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int s = 8 * cc + e, S = s >> 4;
                            const float f = S < R ? rowf[S] * colf[s] : (S == R ? dg[s & 15] : 0.f);
                            m[e] = f * x[s];
                        }
                        *reinterpret_cast<uint4*>(smem + TMoff(b) + tc::swz_off(128 + r, cc, 128)) = pack_f16x8(m);
                    }
                }
                const float gl = vb[63];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int idx = it + 128 * u, rr = idx >> 4, cc = idx & 15, hf = cc >> 3, c8 = cc & 7;
                    float kx[8];
                    unpack_f16x8(*reinterpret_cast<const uint4*>(smem + Xoff(b) + hf * 16384 + tc::swz_off(rr, c8, 128)), kx);
                    const float f = expf(gl - vb[rr]);
#pragma unroll
                    for (int e = 0; e < 8; ++e) kx[e] *= f;
                    *reinterpret_cast<uint4*>(smem + KGoff(b) + hf * 8192 + tc::swz_off(rr, c8, 128)) = pack_f16x8(kx);
                }
            }
            tc::bar_sync(BID, 128);

            // ---- T = (I + A)^-1: 16x16 diagonal blocks by forward substitution ----------------
            {
                const int w4 = warp - 4;
                if (lane < 16) {
                    const int b0 = w4 * 16, j = lane;
                    float xs[16];
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
                        for (int s = 0; s < r; ++s) acc -= fA[(b0 + r) * 65 + b0 + s] * xs[s];
                        xs[r] = acc;
                    }
#pragma unroll
                    for (int r = 0; r < 16; ++r) fT[(b0 + r) * 65 + b0 + j] = xs[r];
                }
            }
            tc::bar_sync(BID, 128);
            // off-diagonal blocks, d = i - j = 1, 2, 3:  T_ij = -T_ii sum_{m=j}^{i-1} A_im T_mj
            for (int d = 1; d < 4; ++d) {
                const int nblk = 4 - d;
                for (int o = it; o < nblk * 256; o += 128) {
                    const int blk = o >> 8, i = d + blk, j = i - d, e = o & 255, rr = e >> 4, cc = e & 15;
                    float acc = 0.f;
                    for (int m = j; m < i; ++m) {
#pragma unroll
                        for (int s = 0; s < 16; ++s) acc += fA[(16 * i + rr) * 65 + 16 * m + s] * fT[(16 * m + s) * 65 + 16 * j + cc];
                    }
                    fZ[(blk * 16 + rr) * 17 + cc] = acc;
                }
                tc::bar_sync(BID, 128);
                for (int o = it; o < nblk * 256; o += 128) {
                    const int blk = o >> 8, i = d + blk, j = i - d, e = o & 255, rr = e >> 4, cc = e & 15;
                    float acc = 0.f;
#pragma unroll
                    for (int s = 0; s < 16; ++s)
                        if (s <= rr) acc -= fT[(16 * i + rr) * 65 + 16 * i + s] * fZ[(blk * 16 + s) * 17 + cc];
                    fT[(16 * i + rr) * 65 + 16 * j + cc] = acc;
                }
                tc::bar_sync(BID, 128);
            }
            // T_u = T diag(beta), T_w = T diag(beta Gamma): fp16 rows 0-63 / 64-127 of [T_u; T_w; M]
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int idx = it + 128 * u, which = idx >> 9, r = (idx >> 3) & 63, cc = idx & 7;
                float t8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = 8 * cc + e;
                    const float sc = which ? vb[128 + s] * vb[64 + s] : vb[128 + s];
                    t8[e] = s <= r ? fT[r * 65 + s] * sc : 0.f;
                }
                *reinterpret_cast<uint4*>(smem + TMoff(b) + tc::swz_off(which * 64 + r, cc, 128)) = pack_f16x8(t8);
            }
            operands_ready();

            // ---- U~ = T_u V_slab (into this slot's TMEM columns) and W = T_w K ------------------
            if (it == 0) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t at = tc::smem_desc(sTM + kk * 32, 16, 1024, tc::kSw128);
                    const uint64_t bv = tc::smem_desc(sVS + kk * 16 * Cf::ROWB, 64 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
                    tc::mma_f16(tmem + Cf::COL_UT + b * NS, at, bv, id_slab, kk > 0);
                    const uint64_t bk = tc::smem_desc(sX + kk * 2048, 16384, 1024, tc::kSw128);
                    tc::mma_f16(tmem + Cf::COL_W, at, bk, id_w, kk > 0);
                }
            }
            if (!(ok = commit_wait())) break;

            // ---- W -> rows 0-63 of this slot's [W;Q] ----------------------------------------------
            if (it >= 64) {
                const int r = it - 64;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float w[32];
                    tc::tmem_ld32(trow + Cf::COL_W + 32 * q4, w);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const int ch = q4 * 4 + cc;
                        *reinterpret_cast<uint4*>(smem + Xoff(b) + (ch >> 3) * 16384 + tc::swz_off(r, ch & 7, 128)) =
                            pack_f16x8(w + 8 * cc);
                    }
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::bar_sync(BID, 128);
            if (it == 0) tc::mbar_arrive(bar_full + b);  // hand slot b to the chain group
        }
        (void)ok;
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, Cf::TMEM_COLS);
    }
}

template <int NS>
inline cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t st) {
    using Cf = TcCfg<NS>;
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_tc_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::BYTES);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(a.num_seqs * a.H * (128 / NS));
    chunk_fwd_tc_kernel<NS><<<grid, 256, Cf::BYTES, st>>>(a);
    return cudaGetLastError();
}

inline cudaError_t chunk_tc_launch(const ChunkArgs& a, cudaStream_t st, const char** why) {
    *why = nullptr;
    if (a.chunk != 64) {
        *why = "only chunk = 64 is built";
        return cudaSuccess;
    }
    // 32-column slabs give 4 CTAs per (sequence, head); use 64-column slabs when that
    // would not fit the GPU's 148 SMs in one wave.
    const long long units = (long long)a.num_seqs * a.H;
    if (units * 4 <= 148) return launch_chunk_tc<32>(a, st);
    return launch_chunk_tc<64>(a, st);
}

}  // namespace gdn
