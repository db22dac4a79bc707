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
// Every decay factor is exp(<= 0): the masks are applied elementwise to the fp32
// products in the TMEM epilogue, never factored as Gamma_r / Gamma_s.
//
// Work decomposition.  The dv columns of S evolve independently (W and A do not depend
// on V), so one CTA owns one (sequence, head, dv-slab of NS columns) and walks the
// sequence chunk by chunk with its slab of S resident in registers (fp32 master copy) and
// in shared memory (fp16 tensor-core operand).  Every product runs on tcgen05 with fp16
// operands and fp32 accumulation in TMEM:
//     [K;Q] K^T            (M=128, N=64,  K=128)   -> A (rows 0-63) and M (rows 64-127)
//     [T_u;T_w] V_slab     (M=128, N=NS,  K=64)    -> U~ (rows 0-63)
//     [T_u;T_w] K          (M=128, N=128, K=64)    -> W  (rows 64-127)
//     [W;Q] S              (M=128, N=NS,  K=128)   -> W S (rows 0-63), Q S (rows 64-127)
//     [T_w;M] U            (M=128, N=NS,  K=64)    -> M U (rows 64-127)
//     (diag(Gamma_C/Gamma)K)^T U (M=128, N=NS, K=64) -> state increment
// with T_u = T diag(beta), T_w = T diag(beta Gamma).  The 64x64 unit-lower-triangular
// inverse T is formed in fp32 on the CUDA cores (16x16 diagonal blocks by forward
// substitution, then the off-diagonal blocks in three dependent rounds).
// Shared-memory operand tiles use the 128B (or 64B) swizzled canonical layouts, so one
// tile (K or the slab tiles) serves both as a K-major and as an MN-major operand.
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
    static constexpr int ROWB = NS * 2;                          // bytes per row of a slab tile
    static constexpr uint32_t SWZ = NS == 32 ? tc::kSw64 : tc::kSw128;
    static constexpr int OFF_QK = 0;                             // [K;Q] / [W;Q]: 2 x [128 x 128 B]
    static constexpr int OFF_KG = OFF_QK + 32768;                // Kg: 2 x [64 x 128 B]
    static constexpr int OFF_T = OFF_KG + 16384;                 // [T_u; T_w; M]: [192 x 128 B]
    static constexpr int OFF_V = OFF_T + 24576;                  // V slab [64 x ROWB]
    static constexpr int OFF_U = OFF_V + 64 * ROWB;              // U [64 x ROWB]
    static constexpr int OFF_S = OFF_U + 64 * ROWB;              // S operand [128 x ROWB]
    static constexpr int OFF_A = OFF_S + 128 * ROWB;             // fp32 A [64][65]
    static constexpr int OFF_TF = OFF_A + 64 * 65 * 4;           // fp32 T [64][65]
    static constexpr int OFF_Z = OFF_TF + 64 * 65 * 4;           // fp32 scratch [3][16][17]
    static constexpr int OFF_VEC = OFF_Z + 3 * 16 * 17 * 4;      // gamma[64], Gamma[64], beta[64]
    static constexpr int OFF_BAR = OFF_VEC + 3 * 64 * 4;         // mbarrier + TMEM base
    static constexpr int BYTES = OFF_BAR + 64 + 1024;            // + alignment slack
    // TMEM columns (fp32 accumulators, lane = output row)
    static constexpr uint32_t COL_QK = 0, COL_UT = 64, COL_W = 128, COL_1 = 256, COL_MU = 256 + NS,
                              COL_DS = 256 + 2 * NS;
    static constexpr uint32_t TMEM_COLS = 512;
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

template <int NS>
__global__ void __launch_bounds__(128, 1) chunk_fwd_tc_kernel(const __grid_constant__ ChunkArgs a) {
    using Cf = TcCfg<NS>;
    constexpr int C = Cf::C;
    constexpr int NSLAB = 128 / NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = tc::smem_u32(smem);
    const uint32_t sQK = sbase + Cf::OFF_QK, sKG = sbase + Cf::OFF_KG, sT = sbase + Cf::OFF_T;
    const uint32_t sV = sbase + Cf::OFF_V, sU = sbase + Cf::OFF_U, sS = sbase + Cf::OFF_S;
    float* fA = reinterpret_cast<float*>(smem + Cf::OFF_A);
    float* fT = reinterpret_cast<float*>(smem + Cf::OFF_TF);
    float* fZ = reinterpret_cast<float*>(smem + Cf::OFF_Z);
    float* s_gam = reinterpret_cast<float*>(smem + Cf::OFF_VEC);
    float* s_Gam = s_gam + 64;
    float* s_beta = s_gam + 128;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cf::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::OFF_BAR + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slab = blockIdx.x % NSLAB;
    const int h = (blockIdx.x / NSLAB) % a.H;
    const int n = blockIdx.x / (NSLAB * a.H);
    const int H = a.H;
    int t_begin, t_end;
    seq_bounds(a.cu, n, a.num_seqs, a.N, t_begin, t_end);

    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, Cf::TMEM_COLS);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's TMEM lanes
    uint32_t phase = 0;
    bool ok = true;

    // Issue-side helpers (thread 0 issues, every thread waits for the commit).
    auto commit_wait = [&]() -> bool {
        if (tid == 0) tc::mma_commit(bar);
        bool w = tc::mbar_wait_bounded(bar, phase, a.budget);
        w = __syncthreads_and(w) != 0;
        if (!w) {
            if (tid == 0) raise_error(kErrTimeout);
            tc::mbar_wait_bounded(bar, phase, 4000000000ull);  // let the MMAs drain before teardown
        }
        phase ^= 1u;
        tc::tc_fence_after();
        return w;
    };
    auto operands_ready = [&]() {  // generic-proxy smem writes + TMEM reads done -> MMA may run
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
    };

    // ---- initial state: thread t owns state row i = t of the slab -----------------------
    const size_t st_base = ((size_t)n * H + h) * 128 * 128 + (size_t)tid * 128 + slab * NS;
    float S[NS];
#pragma unroll
    for (int j = 0; j < NS; j += 4) {
        float4 v4 = a.S0 ? *reinterpret_cast<const float4*>(a.S0 + st_base + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
    }
#pragma unroll
    for (int c = 0; c < NS / 8; ++c)
        *reinterpret_cast<uint4*>(smem + Cf::OFF_S + tc::swz_off(tid, c, Cf::ROWB)) = pack_f16x8(S + 8 * c);

    const uint32_t id_qk = tc::idesc_f16(128, 64, false, false);
    const uint32_t id_slab = tc::idesc_f16(128, NS, false, true);
    const uint32_t id_w = tc::idesc_f16(128, 128, false, true);
    const uint32_t id_ds = tc::idesc_f16(128, NS, true, true);

    float keep[NS];  // rows 0-63: U~ row; rows 64-127: (Q S) row

    for (int c0 = t_begin; c0 < t_end && ok; c0 += C) {
        const int L = min(C, t_end - c0);

        // ---- 1. stage K, Q (fp16, rows 0-63 / 64-127 of [K;Q]) and the V slab ------------
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int idx = tid + 128 * u, r = idx >> 4, cc = idx & 15;
            uint4 kv = make_uint4(0, 0, 0, 0), qv = kv;
            if (r < L) {
                const size_t off = ((size_t)(c0 + r) * H + h) * 128 + cc * 8;
                kv = to_f16x8(*reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.k) + off), a.in_dt);
                qv = to_f16x8(*reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.q) + off), a.in_dt);
            }
            const int hf = cc >> 3, c8 = cc & 7;
            *reinterpret_cast<uint4*>(smem + Cf::OFF_QK + hf * 16384 + tc::swz_off(r, c8, 128)) = kv;
            *reinterpret_cast<uint4*>(smem + Cf::OFF_QK + hf * 16384 + tc::swz_off(r + 64, c8, 128)) = qv;
        }
#pragma unroll
        for (int u = 0; u < (64 * NS / 8) / 128; ++u) {
            const int idx = tid + 128 * u, r = idx / (NS / 8), cc = idx % (NS / 8);
            uint4 vv = make_uint4(0, 0, 0, 0);
            if (r < L) {
                const size_t off = ((size_t)(c0 + r) * H + h) * 128 + slab * NS + cc * 8;
                vv = to_f16x8(*reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.v) + off), a.in_dt);
            }
            *reinterpret_cast<uint4*>(smem + Cf::OFF_V + tc::swz_off(r, cc, Cf::ROWB)) = vv;
        }
        // ---- 2. gates: gamma = inclusive prefix sum of g inside the chunk ---------------
        if (tid < 64) {
            const bool valid = tid < L;
            float gv = valid ? a.g[(size_t)(c0 + tid) * H + h] : 0.f;
            s_beta[tid] = valid ? a.beta[(size_t)(c0 + tid) * H + h] : 0.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, gv, o);
                if (lane >= o) gv += y;
            }
            s_gam[tid] = gv;
        }
        __syncthreads();
        if (tid >= 32 && tid < 64) s_gam[tid] += s_gam[31];
        __syncthreads();
        if (tid < 64) s_Gam[tid] = expf(s_gam[tid]);
        operands_ready();

        // ---- 3. [K;Q] K^T ------------------------------------------------------------------
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint64_t d = tc::smem_desc(sQK + off, 16, 1024, tc::kSw128);
                tc::mma_f16(tmem + Cf::COL_QK, d, d, id_qk, kk > 0);
            }
        }
        if (!(ok = commit_wait())) break;

        // ---- 4. masks: A (fp32, for the solve) and M (fp16 operand); Kg -------------------
        {
            float x[64];
            tc::tmem_ld32(trow + Cf::COL_QK, x);
            tc::tmem_ld32(trow + Cf::COL_QK + 32, x + 32);
            if (tid < 64) {
                const int r = tid;
                const float gr = s_gam[r], br = s_beta[r];
#pragma unroll
                for (int s = 0; s < 64; ++s) fA[r * 65 + s] = s < r ? br * expf(gr - s_gam[s]) * x[s] : 0.f;
            } else {
                const int r = tid - 64;
                const float gr = s_gam[r];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float m[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int s = 8 * c + e;
                        m[e] = s <= r ? expf(gr - s_gam[s]) * x[s] : 0.f;
                    }
                    *reinterpret_cast<uint4*>(smem + Cf::OFF_T + tc::swz_off(128 + r, c, 128)) = pack_f16x8(m);
                }
            }
            const float gl = s_gam[63];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int idx = tid + 128 * u, r = idx >> 4, cc = idx & 15, hf = cc >> 3, c8 = cc & 7;
                float kx[8];
                unpack_f16x8(*reinterpret_cast<const uint4*>(smem + Cf::OFF_QK + hf * 16384 + tc::swz_off(r, c8, 128)), kx);
                const float f = expf(gl - s_gam[r]);
#pragma unroll
                for (int e = 0; e < 8; ++e) kx[e] *= f;
                *reinterpret_cast<uint4*>(smem + Cf::OFF_KG + hf * 8192 + tc::swz_off(r, c8, 128)) = pack_f16x8(kx);
            }
        }
        __syncthreads();

        // ---- 5. T = (I + A)^-1: 16x16 diagonal blocks by forward substitution --------------
        if (lane < 16) {
            const int b0 = warp * 16, j = lane;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
                for (int s = 0; s < r; ++s) acc -= fA[(b0 + r) * 65 + b0 + s] * x[s];
                x[r] = acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) fT[(b0 + r) * 65 + b0 + j] = x[r];
        }
        __syncthreads();
        // off-diagonal blocks, d = i - j = 1, 2, 3:  T_ij = -T_ii sum_{m=j}^{i-1} A_im T_mj
        for (int d = 1; d < 4; ++d) {
            const int nblk = 4 - d;
            for (int o = tid; o < nblk * 256; o += 128) {
                const int blk = o >> 8, i = d + blk, j = i - d, e = o & 255, rr = e >> 4, cc = e & 15;
                float acc = 0.f;
                for (int m = j; m < i; ++m) {
#pragma unroll
                    for (int s = 0; s < 16; ++s) acc += fA[(16 * i + rr) * 65 + 16 * m + s] * fT[(16 * m + s) * 65 + 16 * j + cc];
                }
                fZ[(blk * 16 + rr) * 17 + cc] = acc;
            }
            __syncthreads();
            for (int o = tid; o < nblk * 256; o += 128) {
                const int blk = o >> 8, i = d + blk, j = i - d, e = o & 255, rr = e >> 4, cc = e & 15;
                float acc = 0.f;
#pragma unroll
                for (int s = 0; s < 16; ++s)
                    if (s <= rr) acc -= fT[(16 * i + rr) * 65 + 16 * i + s] * fZ[(blk * 16 + s) * 17 + cc];
                fT[(16 * i + rr) * 65 + 16 * j + cc] = acc;
            }
            __syncthreads();
        }
        // T_u = T diag(beta), T_w = T diag(beta Gamma) as fp16 operands (rows 0-63 / 64-127)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int idx = tid + 128 * u, which = idx >> 9, r = (idx >> 3) & 63, c = idx & 7;
            float t8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int s = 8 * c + e;
                const float sc = which ? s_beta[s] * s_Gam[s] : s_beta[s];
                t8[e] = s <= r ? fT[r * 65 + s] * sc : 0.f;
            }
            *reinterpret_cast<uint4*>(smem + Cf::OFF_T + tc::swz_off(which * 64 + r, c, 128)) = pack_f16x8(t8);
        }
        operands_ready();

        // ---- 6. U~ = T_u V_slab and W = T_w K ----------------------------------------------
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t at = tc::smem_desc(sT + kk * 32, 16, 1024, tc::kSw128);
                const uint64_t bv = tc::smem_desc(sV + kk * 16 * Cf::ROWB, 64 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
                tc::mma_f16(tmem + Cf::COL_UT, at, bv, id_slab, kk > 0);
                const uint64_t bk = tc::smem_desc(sQK + kk * 2048, 16384, 1024, tc::kSw128);
                tc::mma_f16(tmem + Cf::COL_W, at, bk, id_w, kk > 0);
            }
        }
        if (!(ok = commit_wait())) break;

        // ---- 7. W -> rows 0-63 of the [W;Q] operand; U~ kept in registers -------------------
        if (tid >= 64) {
            const int r = tid - 64;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float w[32];
                tc::tmem_ld32(trow + Cf::COL_W + 32 * q4, w);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int cc = q4 * 4 + c;  // 16-byte chunk 0..15 of the 128-wide row
                    *reinterpret_cast<uint4*>(smem + Cf::OFF_QK + (cc >> 3) * 16384 + tc::swz_off(r, cc & 7, 128)) =
                        pack_f16x8(w + 8 * c);
                }
            }
        } else {
#pragma unroll
            for (int q4 = 0; q4 < NS / 32; ++q4) tc::tmem_ld32(trow + Cf::COL_UT + 32 * q4, keep + 32 * q4);
        }
        operands_ready();

        // ---- 8. [W;Q] S ---------------------------------------------------------------------
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t aw = tc::smem_desc(sQK + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, tc::kSw128);
                const uint64_t bs = tc::smem_desc(sS + kk * 16 * Cf::ROWB, 128 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
                tc::mma_f16(tmem + Cf::COL_1, aw, bs, id_slab, kk > 0);
            }
        }
        if (!(ok = commit_wait())) break;

        // ---- 9. U = U~ - W S (fp16 operand); Q S kept -----------------------------------------
        {
            float d1[NS];
#pragma unroll
            for (int q4 = 0; q4 < NS / 32; ++q4) tc::tmem_ld32(trow + Cf::COL_1 + 32 * q4, d1 + 32 * q4);
            if (tid < 64) {
#pragma unroll
                for (int j = 0; j < NS; ++j) d1[j] = keep[j] - d1[j];
#pragma unroll
                for (int c = 0; c < NS / 8; ++c)
                    *reinterpret_cast<uint4*>(smem + Cf::OFF_U + tc::swz_off(tid, c, Cf::ROWB)) = pack_f16x8(d1 + 8 * c);
            } else {
#pragma unroll
                for (int j = 0; j < NS; ++j) keep[j] = d1[j];
            }
        }
        operands_ready();

        // ---- 10. M U (into rows 64-127) and Kg^T U ------------------------------------------
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bu = tc::smem_desc(sU + kk * 16 * Cf::ROWB, 64 * Cf::ROWB, 8 * Cf::ROWB, Cf::SWZ);
                const uint64_t am = tc::smem_desc(sT + 64 * 128 + kk * 32, 16, 1024, tc::kSw128);
                tc::mma_f16(tmem + Cf::COL_MU, am, bu, id_slab, kk > 0);
                const uint64_t ak = tc::smem_desc(sKG + kk * 2048, 8192, 1024, tc::kSw128);
                tc::mma_f16(tmem + Cf::COL_DS, ak, bu, id_ds, kk > 0);
            }
        }
        if (!(ok = commit_wait())) break;

        // ---- 11. Y = Gamma (Q S) + M U; S <- Gamma_C S + Kg^T U ------------------------------
        {
            float t[NS];
            if (tid >= 64) {
                const int r = tid - 64;
#pragma unroll
                for (int q4 = 0; q4 < NS / 32; ++q4) tc::tmem_ld32(trow + Cf::COL_MU + 32 * q4, t + 32 * q4);
                if (r < L) {
                    const float gr = s_Gam[r];
                    const size_t yoff = ((size_t)(c0 + r) * H + h) * 128 + slab * NS;
#pragma unroll
                    for (int j = 0; j < NS; j += 4)
                        st4(a.y, a.y_dt, yoff + j,
                            make_float4(a.scale * (gr * keep[j] + t[j]), a.scale * (gr * keep[j + 1] + t[j + 1]),
                                        a.scale * (gr * keep[j + 2] + t[j + 2]), a.scale * (gr * keep[j + 3] + t[j + 3])));
                }
            } else {
#pragma unroll
                for (int q4 = 0; q4 < NS / 32; ++q4) tc::tmem_ld32(trow + Cf::COL_MU + 32 * q4, t + 32 * q4);  // keep warps converged
            }
#pragma unroll
            for (int q4 = 0; q4 < NS / 32; ++q4) tc::tmem_ld32(trow + Cf::COL_DS + 32 * q4, t + 32 * q4);
            const float gC = s_Gam[63];
#pragma unroll
            for (int j = 0; j < NS; ++j) S[j] = gC * S[j] + t[j];
#pragma unroll
            for (int c = 0; c < NS / 8; ++c)
                *reinterpret_cast<uint4*>(smem + Cf::OFF_S + tc::swz_off(tid, c, Cf::ROWB)) = pack_f16x8(S + 8 * c);
        }
        operands_ready();
    }

    if (ok && a.S_T) {
#pragma unroll
        for (int j = 0; j < NS; j += 4)
            *reinterpret_cast<float4*>(a.S_T + st_base + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
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
    chunk_fwd_tc_kernel<NS><<<grid, 128, Cf::BYTES, st>>>(a);
    return cudaGetLastError();
}

inline cudaError_t chunk_tc_launch(const ChunkArgs& a, cudaStream_t st, const char** why) {
    *why = nullptr;
    if (a.chunk != 64) {
        *why = "only chunk = 64 is built";
        return cudaSuccess;
    }
    // 32-column slabs give 4 CTAs per (sequence, head); use 64-column slabs when that
    // already covers the GPU.
    const long long units = (long long)a.num_seqs * a.H;
    if (units * 4 <= 148) return launch_chunk_tc<32>(a, st);
    return launch_chunk_tc<64>(a, st);
}

}  // namespace gdn
