// inproj.cuh -- the mixer's input projections fused with eqs. (6)-(10) of "On the design of
// Qwen3.8-Next architecture", section 2.1.1 ("GDN parameterisation").
//
// From the normalised residual stream x_t (D channels) the mixer forms W_q x_t, W_k x_t,
// W_v x_t (the ShortConv inputs of eqs. 6-8), W_beta x_t and W_alpha x_t (the gate logits of
// eqs. 9-10) and W_z x_t (the output gate of eq. 11).  All six are one product
// P = x W^T with W = [W_q; W_k; W_v; W_z; W_beta; W_alpha] stacked as rows, a dense
// contraction over D, so it runs on the tcgen05 tensor cores; the elementwise steps that
// follow run in the epilogue on the fp32 accumulators, and the raw projections never reach
// HBM.
//
// inproj_prep_kernel is persistent: one CTA per SM walks the output tiles.  A tile is 128
// consecutive tokens by 256 output channels (two heads of d = 128), or by the 2H gate-logit
// channels for the gate tile of each token block.  ShortConv at token t reads tokens
// t-(TAPS-1) .. t, so a tile's first TAPS-1 rows are a halo: they are recomputed by the tile
// before, and each tile outputs 128-(TAPS-1) tokens.
//   warp 0      TMA producer: x and W tiles, 64 channels of D (one 128-byte swizzle row) per
//               stage, three stages in flight
//   warp 1      allocates TMEM; one lane issues the MMAs (M = 128, N = 256 or 2H, K = 16) into
//               one of two TMEM accumulators, so the epilogue of a tile overlaps the next
//               tile's products
//   warps 2-9   epilogue, two groups of four warps (two warps per SM sub-partition, so one
//               hides the other's latency).  A thread owns one token (its TMEM lane) and, in
//               group g, channels [64 g, 64 g + 64) of each head.  Conv tiles stage those 64
//               columns in shared memory, where each thread reads its token's TAPS-1
//               predecessors four columns at a time; then SiLU, and for q and k the L2Norm
//               over the head's 128 channels, whose sum of squares the two groups exchange
//               through shared memory.  v: conv and SiLU.  z: stored as is.  Results go back
//               through the staging rows in 16-bit form so that each warp stores whole 128-byte
//               row segments.  Gate tile: beta = sigmoid (eq. 9), g = -exp(A_h) softplus(. + b_h)
//               (eq. 10).
// Every wait is bounded: a wait that runs out flags kErrTimeout and then waits for the
// hardware event (a TMA copy or an MMA always completes), so every role walks the same tiles
// and the CTA always reaches its teardown.
#pragma once
#include "common.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace gdn {

template <int TAPS>
struct IpCfg {
    static constexpr int BM = 128, BN = 256, BK = 64, STAGES = 3;
    static constexpr int HALO = TAPS - 1, ROWS_OUT = BM - HALO;
    static constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE = A_BYTES + B_BYTES;
    static constexpr int XC = 64, XLD = XC + 4;                   // staged columns, row stride (floats)
    static constexpr int OFF_X = STAGES * STAGE;                  // per group [BM][XLD] fp32
    static constexpr int OFF_TAPS = OFF_X + 2 * BM * XLD * 4;     // [BN][TAPS] fp32, right-aligned
    static constexpr int OFF_SS = OFF_TAPS + BN * TAPS * 4;       // [2 heads][2 groups][BM] sums of squares
    static constexpr int OFF_BAR = OFF_SS + 4 * BM * 4;           // full[S], empty[S], accf[2], acce[2]
    static constexpr int NBAR = 2 * STAGES + 4;
    static constexpr int OFF_SLOT = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_SLOT + 16;
    static constexpr int ALIGN = 1024;                            // 128-byte swizzle atoms
    static constexpr int THREADS = 320;
    static constexpr int EPI_WARPS = 8;
    static constexpr int TMEM_COLS = 512;                         // two 256-column accumulators
    static_assert(BYTES + ALIGN <= 232448, "shared memory");
    static_assert(OFF_X % 16 == 0 && OFF_TAPS % 16 == 0 && OFF_SS % 16 == 0 && OFF_BAR % 8 == 0, "alignment");
};

struct InprojArgs {
    int N, D, H, W;              // tokens, model width, heads, conv taps (<= TAPS)
    int nq;                      // 256-channel tiles per projection (H * 128 / 256)
    int n_tiles_n;               // tiles per token block: 3 nq (+ nq with z) + 1
    int has_z;
    long long n_tiles;           // token blocks x n_tiles_n
    const float* conv_q;         // [H*128, W]
    const float* conv_k;
    const float* conv_v;
    const float* A_log;          // [H]
    const float* alpha_bias;     // [H]
    const int32_t* cu;
    int num_seqs;
    float eps;
    int out_dt;                  // kBF16 or kF16: q, k, v, z
    void* q;
    void* k;
    void* v;
    void* z;
    float* g;
    float* beta;
    unsigned long long budget;
};

struct InprojMaps {
    CUtensorMap x;      // [N, D], box 64 x 128
    CUtensorMap w;      // [4 H 128 + 2H, D], box 64 x 256
    CUtensorMap wg;     // same rows, box 64 x 2H (the gate rows)
};

namespace ip {

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            tc::smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(tc::smem_u32(bar))
        : "memory");
}

// Warp-wide load of 16 consecutive fp32 columns of the warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// The same load without the wait, so that several can be in flight; tmem_wait() completes them.
__device__ __forceinline__ void tmem_ld16_nw(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 64 consecutive accumulator columns of the warp's lanes into v.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
    uint32_t u[64];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld16_nw(taddr + 16 * c, u + 16 * c);
    tmem_wait();
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(u[i]);
}

__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); }

// A bounded wait that, once it runs out, flags the error and then waits for the event itself.
__device__ __forceinline__ void wait(uint64_t* bar, uint32_t parity, unsigned long long budget) {
    if (!tc::mbar_wait_bounded(bar, parity, budget)) {
        raise_error(kErrTimeout);
        tc::mbar_wait_bounded(bar, parity, 4000000000ull);
    }
}

// Tile kinds by column-tile index within a token block.
enum Kind : int { kQ = 0, kK = 1, kV = 2, kZ = 3, kGate = 4 };

__device__ __forceinline__ void tile_of(const InprojArgs& a, long long tile, int& mt, int& kind, int& local) {
    mt = (int)(tile / a.n_tiles_n);
    const int nt = (int)(tile - (long long)mt * a.n_tiles_n);
    const int nconv = (3 + a.has_z) * a.nq;
    if (nt >= nconv) {
        kind = kGate;
        local = 0;
    } else {
        kind = nt / a.nq;
        local = nt - kind * a.nq;
    }
}

// 8 values -> 16 bytes of 16-bit storage
__device__ __forceinline__ uint4 pack8(const float* x, bool bf) {
    uint4 u;
    if (bf) {
        u.x = pack2<true>(x[0], x[1]); u.y = pack2<true>(x[2], x[3]);
        u.z = pack2<true>(x[4], x[5]); u.w = pack2<true>(x[6], x[7]);
    } else {
        u.x = pack2<false>(x[0], x[1]); u.y = pack2<false>(x[2], x[3]);
        u.z = pack2<false>(x[4], x[5]); u.w = pack2<false>(x[6], x[7]);
    }
    return u;
}

}  // namespace ip

template <bool BF, int TAPS>
__global__ void __launch_bounds__(IpCfg<TAPS>::THREADS, 1)
inproj_prep_kernel(const __grid_constant__ InprojMaps maps, const InprojArgs a) {
    using Cf = IpCfg<TAPS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + Cf::ALIGN - 1) &
                                               ~(uintptr_t)(Cf::ALIGN - 1));
    const uint32_t sbase = tc::smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cf::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = bars + Cf::STAGES;
    uint64_t* accf = bars + 2 * Cf::STAGES;
    uint64_t* acce = accf + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cf::OFF_SLOT);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int KB = a.D / Cf::BK;

    if (tid == 0) {
        for (int i = 0; i < Cf::NBAR; ++i) tc::mbar_init(bars + i, i >= 2 * Cf::STAGES + 2 ? Cf::EPI_WARPS : 1);
        tc::fence_mbar_init();
        tc::prefetch_tmap(&maps.x);
        tc::prefetch_tmap(&maps.w);
        tc::prefetch_tmap(&maps.wg);
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, Cf::TMEM_COLS);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ================================ TMA producer ================================
        if (lane == 0) {
            int stage = 0;
            uint32_t ph = 0;
            for (long long tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x) {
                int mt, kind, local;
                ip::tile_of(a, tile, mt, kind, local);
                const int row0 = mt * Cf::ROWS_OUT - Cf::HALO;  // may be negative: zero fill
                const int wrow0 = kind == ip::kGate ? 4 * a.H * 128 : kind * a.H * 128 + local * Cf::BN;
                const uint32_t bytes = Cf::A_BYTES + (kind == ip::kGate ? 2 * a.H : Cf::BN) * Cf::BK * 2;
                for (int kb = 0; kb < KB; ++kb) {
                    ip::wait(empty + stage, ph ^ 1u, a.budget);
                    uint8_t* sa = smem + stage * Cf::STAGE;
                    tc::mbar_arrive_expect_tx(full + stage, bytes);
                    ip::tma_load_2d(sa, &maps.x, kb * Cf::BK, row0, full + stage);
                    ip::tma_load_2d(sa + Cf::A_BYTES, kind == ip::kGate ? (const void*)&maps.wg : (const void*)&maps.w,
                                    kb * Cf::BK, wrow0, full + stage);
                    if (++stage == Cf::STAGES) {
                        stage = 0;
                        ph ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ==================================
        if (lane == 0) {
            int stage = 0;
            uint32_t ph = 0;
            int it = 0;
            const uint64_t dA0 = tc::smem_desc(sbase, 16, 1024, tc::kSw128);
            const uint64_t dB0 = tc::smem_desc(sbase + Cf::A_BYTES, 16, 1024, tc::kSw128);
            for (long long tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, ++it) {
                int mt, kind, local;
                ip::tile_of(a, tile, mt, kind, local);
                const int buf = it & 1;
                const uint32_t use = (uint32_t)(it >> 1);
                const uint32_t idesc = BF ? tc::idesc_bf16(128, kind == ip::kGate ? 2 * a.H : Cf::BN, false, false)
                                          : tc::idesc_f16(128, kind == ip::kGate ? 2 * a.H : Cf::BN, false, false);
                ip::wait(acce + buf, (use & 1u) ^ 1u, a.budget);
                tc::tc_fence_after();
                const uint32_t d = tmem + buf * 256;
                for (int kb = 0; kb < KB; ++kb) {
                    ip::wait(full + stage, ph, a.budget);
                    tc::tc_fence_after();
                    const uint64_t da = ip::desc_add(dA0, stage * Cf::STAGE), db = ip::desc_add(dB0, stage * Cf::STAGE);
#pragma unroll
                    for (int kk = 0; kk < Cf::BK / 16; ++kk)
                        tc::mma_f16(d, ip::desc_add(da, kk * 32), ip::desc_add(db, kk * 32), idesc, (kb | kk) != 0);
                    tc::mma_commit(empty + stage);
                    if (++stage == Cf::STAGES) {
                        stage = 0;
                        ph ^= 1u;
                    }
                }
                tc::mma_commit(accf + buf);
            }
        }
    } else {
        // ================================ epilogue ====================================
        const int grp = (warp - 2) >> 2;           // column group: channels [64 grp, 64 grp + 64) of a head
        const int quad = warp & 3;                 // TMEM lanes 32 quad .. 32 quad + 31
        const int r = quad * 32 + lane;            // this thread's tile row
        const int gt = (warp - 2 - 4 * grp) * 32 + lane;  // 0..127 within the group
        const int BIDG = 1 + grp;                  // named barrier of the group's 128 threads
        constexpr int BID_PAIR = 3;                // both groups (the sum-of-squares exchange)
        float* X = reinterpret_cast<float*>(smem + Cf::OFF_X) + grp * Cf::BM * Cf::XLD;
        float* taps = reinterpret_cast<float*>(smem + Cf::OFF_TAPS);
        float* ssx = reinterpret_cast<float*>(smem + Cf::OFF_SS);
        const int stop = a.cu ? min(max(a.cu[a.num_seqs], 0), a.N) : (a.N / a.num_seqs) * a.num_seqs;
        const bool bf_out = a.out_dt == kBF16;
        const size_t HD = (size_t)a.H * 128;
        if (blockIdx.x == 0 && warp == 2 && a.cu != nullptr) {
            // cu_seqlens must be non-decreasing inside [0, N]; a malformed array is flagged (it
            // cannot send an access out of bounds: taps only read rows of the tile)
            bool bad = false;
            for (int m = lane; m < a.num_seqs; m += 32) bad |= a.cu[m] < 0 || a.cu[m + 1] < a.cu[m] || a.cu[m + 1] > a.N;
            if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(kErrSeqlens);
        }
        int it = 0;
        for (long long tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, ++it) {
            int mt, kind, local;
            ip::tile_of(a, tile, mt, kind, local);
            const int buf = it & 1;
            const uint32_t use = (uint32_t)(it >> 1);
            const int tok0 = mt * Cf::ROWS_OUT - Cf::HALO;
            const int t = tok0 + r;
            const bool row_out = r >= Cf::HALO && t < a.N;          // this tile outputs token t
            const bool conv_out = row_out && t < stop;               // ... and t lies in a sequence
            const uint32_t tcol = tmem + ((uint32_t)(quad * 32) << 16) + buf * 256;
            auto release = [&]() {  // every TMEM load of the tile is done: the accumulator is free
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(acce + buf);
            };

            // A warp's 32 rows of 64 16-bit results, written by their owners into the first 128 bytes
            // of their staging rows, leave as whole 128-byte row segments: instruction k stores rows
            // 4k .. 4k+3 of the warp, eight lanes per row.
            auto store_rows = [&](void* base, int col0, int row_end) {  // columns [col0, col0 + 64)
                __syncwarp();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int rr = quad * 32 + 4 * k + (lane >> 3), tt = tok0 + rr;
                    const uint4 u = *reinterpret_cast<const uint4*>(X + rr * Cf::XLD + 4 * (lane & 7));
                    if (rr >= Cf::HALO && tt < row_end && in_bounds(tt, a.N))
                        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(base) +
                                                  ((size_t)tt * HD + (size_t)local * Cf::BN + col0 + 8 * (lane & 7)) * 2) = u;
                }
                __syncwarp();
            };
            auto stage_out = [&](const float* o) {  // this row's 64 results, 16-bit, into its staging row
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) *reinterpret_cast<uint4*>(X + r * Cf::XLD + 4 * c8) = ip::pack8(o + 8 * c8, bf_out);
            };

            if (kind <= ip::kV) {
                // the taps of the group's 128 channels, right-aligned to TAPS (zeros before)
                const float* cw = kind == ip::kQ ? a.conv_q : kind == ip::kK ? a.conv_k : a.conv_v;
                tc::bar_sync(BIDG, 128);  // the group's previous tile no longer reads taps or X
                for (int e = gt; e < 128 * TAPS; e += 128) {
                    const int lc = e / TAPS, i = e - lc * TAPS, j = i - (TAPS - a.W);
                    const int c = (lc >> 6) * 128 + grp * 64 + (lc & 63);
                    taps[c * TAPS + i] = j >= 0 ? __ldg(cw + (size_t)(local * Cf::BN + c) * a.W + j) : 0.f;
                }
            } else if (kind == ip::kZ) {
                tc::bar_sync(BIDG, 128);  // the group's previous tile no longer reads X
            }
            ip::wait(accf + buf, use & 1u, a.budget);
            tc::tc_fence_after();

            if (kind <= ip::kV) {
                int nmask = 0;  // taps before the start of t's sequence read zeros
                if (conv_out) {
                    const int s0 = seq_start_of(a.cu, a.num_seqs, a.N, t);
                    nmask = min(max(s0 - t + Cf::HALO, 0), TAPS);
                }
                const bool clean = __all_sync(0xffffffffu, nmask == 0);  // no masked tap in this warp
                void* outp = kind == ip::kQ ? a.q : kind == ip::kK ? a.k : a.v;
                const bool norm = kind != ip::kV;
                const float* xr = X + (conv_out ? r - Cf::HALO : 0) * Cf::XLD;  // rows t-(TAPS-1) .. t
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    const int col0 = hh * 128 + grp * 64;
                    float v[64];
                    ip::tmem_ld64(tcol + col0, v);
                    if (hh == 1) release();
#pragma unroll
                    for (int c4 = 0; c4 < 16; ++c4)
                        *reinterpret_cast<float4*>(X + r * Cf::XLD + 4 * c4) = make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
                    tc::bar_sync(BIDG, 128);  // the group's rows are staged
                    const float* tp = taps + col0 * TAPS;
#pragma unroll
                    for (int c4 = 0; c4 < 16; ++c4) {
                        float x[TAPS][4];  // rows t-(TAPS-1) .. t of columns 4 c4 .. 4 c4 + 3
#pragma unroll
                        for (int i = 0; i < TAPS - 1; ++i) {
                            const float4 x4 = *reinterpret_cast<const float4*>(xr + i * Cf::XLD + 4 * c4);
                            const bool m = clean || i >= nmask;
                            x[i][0] = m ? x4.x : 0.f; x[i][1] = m ? x4.y : 0.f; x[i][2] = m ? x4.z : 0.f; x[i][3] = m ? x4.w : 0.f;
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j) x[TAPS - 1][j] = v[4 * c4 + j];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float s = 0.f;
#pragma unroll
                            for (int i = 0; i < TAPS; i += 4) {
                                const float4 w4 = *reinterpret_cast<const float4*>(tp + (4 * c4 + j) * TAPS + i);
                                s = fmaf(w4.x, x[i][j], s);
                                s = fmaf(w4.y, x[i + 1][j], s);
                                s = fmaf(w4.z, x[i + 2][j], s);
                                s = fmaf(w4.w, x[i + 3][j], s);
                            }
                            v[4 * c4 + j] = __fdividef(s, 1.0f + __expf(-s));  // SiLU
                        }
                    }
                    float inv = 1.f;
                    if (norm) {  // L2Norm over the head's 128 channels: this group's 64 plus the other's
                        float ss = 0.f;
#pragma unroll
                        for (int j = 0; j < 64; ++j) ss = fmaf(v[j], v[j], ss);
                        ssx[(hh * 2 + grp) * Cf::BM + r] = ss;
                        tc::bar_sync(BID_PAIR, 256);  // also: every row of X has been read by its successors
                        ss += ssx[(hh * 2 + (grp ^ 1)) * Cf::BM + r];
                        inv = rsqrtf(ss + a.eps);
                    } else {
                        tc::bar_sync(BIDG, 128);  // every row of X has been read by its successors
                    }
#pragma unroll
                    for (int j = 0; j < 64; ++j) v[j] *= inv;
                    stage_out(v);
                    store_rows(outp, hh * 128 + grp * 64, stop);
                }
            } else if (kind == ip::kZ) {
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    const int col0 = grp * 128 + hh * 64;
                    float v[64];
                    ip::tmem_ld64(tcol + col0, v);
                    if (hh == 1) release();
                    stage_out(v);
                    store_rows(a.z, col0, a.N);
                }
            } else {
                // gate tile: columns [0, H) beta logits, [H, 2H) alpha logits; group g takes the
                // 16-column chunks g, g + 2, ...
                const int nchunk = (2 * a.H) / 16;
                if (grp >= nchunk) release();
#pragma unroll 1
                for (int cc = grp; cc < nchunk; cc += 2) {
                    float vv[16];
                    ip::tmem_ld16(tcol + cc * 16, vv);
                    if (cc + 2 >= nchunk) release();
                    if (row_out) {
                        // four columns at a time, all beta or all alpha logits (H is a multiple of 16)
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const int c = cc * 16 + 4 * q4;
                            float o[4];
                            if (c < a.H) {
#pragma unroll
                                for (int j = 0; j < 4; ++j) o[j] = 1.0f / (1.0f + expf(-vv[4 * q4 + j]));  // eq. (9)
                                *reinterpret_cast<float4*>(a.beta + (size_t)t * a.H + c) = make_float4(o[0], o[1], o[2], o[3]);
                            } else {
                                const int h = c - a.H;
#pragma unroll
                                for (int j = 0; j < 4; ++j)                                                // eq. (10)
                                    o[j] = -expf(__ldg(a.A_log + h + j)) * softplusf_(vv[4 * q4 + j] + __ldg(a.alpha_bias + h + j));
                                *reinterpret_cast<float4*>(a.g + (size_t)t * a.H + h) = make_float4(o[0], o[1], o[2], o[3]);
                            }
                        }
                    }
                }
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, Cf::TMEM_COLS);
    }
}

// [rows, cols] row-major 16-bit matrix; box = box_cols x box_rows, 128-byte swizzle.
inline bool encode_map_2d(CUtensorMap* m, const void* base, bool bf, long long rows, int cols, uint32_t box_cols,
                          uint32_t box_rows) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gdn
