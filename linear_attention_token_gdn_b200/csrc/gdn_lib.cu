// gdn_lib.cu -- the C ABI of libgdn.so (declared in include/gdn.h): argument validation,
// launch configuration and error reporting around the device kernels.
//
// Every entry point validates on the host and returns before enqueuing anything when an
// argument is wrong; it never synchronises and never allocates.
#include <atomic>
#include <mutex>
#include <vector>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/gdn.h"
#include "common.cuh"
#include "launch_timer.cuh"
#include "decode.cuh"
#include "mixer_decode.cuh"
#include "out_gate.cuh"
#include "prep.cuh"
#include "recurrent.cuh"
#include "state_map.cuh"
#include "bwd.cuh"
#include "chunk_tc.cuh"
#include "inproj.cuh"

namespace {

thread_local char g_msg[256] = "";
std::atomic<unsigned long long> g_wait_budget{0};

gdn_status_t fail(gdn_status_t s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

gdn_status_t launched(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return GDN_OK;
}

bool head_dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool dtype_ok(int t) { return t == GDN_F32 || t == GDN_BF16 || t == GDN_F16; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE(cond, ...)                                            \
    do {                                                              \
        if (!(cond)) return fail(GDN_ERR_INVALID_ARG, __VA_ARGS__);   \
    } while (0)

#define REQUIRE_PTR(p, name)                                                            \
    do {                                                                                \
        if ((p) == nullptr) return fail(GDN_ERR_INVALID_ARG, "%s is NULL", name);       \
        if (!aligned16(p)) return fail(GDN_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
    } while (0)

#define OPT_PTR(p, name)                                                                \
    do {                                                                                \
        if ((p) != nullptr && !aligned16(p))                                            \
            return fail(GDN_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);       \
    } while (0)

// Dispatch a <DK, DV> template over the 16 supported head-size pairs.
template <template <int, int> class F, typename... Args>
gdn_status_t dispatch_dims(int dk, int dv, Args&&... args) {
#define GDN_DV_CASES(DKV)                                                        \
    switch (dv) {                                                                \
        case 16: return F<DKV, 16>::run(args...);                                \
        case 32: return F<DKV, 32>::run(args...);                                \
        case 64: return F<DKV, 64>::run(args...);                                \
        case 128: return F<DKV, 128>::run(args...);                              \
    }                                                                            \
    break;
    switch (dk) {
        case 16: GDN_DV_CASES(16)
        case 32: GDN_DV_CASES(32)
        case 64: GDN_DV_CASES(64)
        case 128: GDN_DV_CASES(128)
    }
#undef GDN_DV_CASES
    return fail(GDN_ERR_INVALID_ARG, "unsupported head sizes dk=%d dv=%d", dk, dv);
}

unsigned long long wait_budget() {
    unsigned long long b = g_wait_budget.load(std::memory_order_relaxed);
    return b ? b : 2000000000ull;  // ~1 s at the B200's boost clock
}

// ---------------------------------------------------------------- launchers

template <int DK, int DV>
struct DecodeLaunch {
    static gdn_status_t run(const void* q, const void* k, const void* v, const float* g, const float* beta,
                            float* state, const int32_t* slot, int num_slots, int B, int H, float scale,
                            int in_dt, int y_dt, void* y, cudaStream_t st) {
        using Sh = gdn::DecodeShape<DK, DV>;
        constexpr int bytes = DK * DV * 4;  // the state block, staged in shared memory
        cudaError_t e = cudaFuncSetAttribute(gdn::decode_step_kernel<DK, DV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "decode_step_kernel smem: %s", cudaGetErrorString(e));
        gdn::LaunchScope timed(st, "decode_step_kernel");
        gdn::decode_step_kernel<DK, DV><<<(unsigned)(B * H), Sh::THREADS, bytes, st>>>(
            q, k, v, g, beta, state, slot, num_slots, H, scale, in_dt, y_dt, y, wait_budget());
        return launched("decode_step_kernel");
    }
};

template <int DK, int DV>
struct MixerDecodeLaunch {
    static gdn_status_t run(const gdn::MixerDecodeArgs& args, int B, cudaStream_t st) {
        using Sh = gdn::DecodeShape<DK, DV>;
        constexpr int bytes = DK * DV * 4;  // the state block, staged in shared memory
        cudaError_t e = args.W <= 4 ? cudaFuncSetAttribute(gdn::mixer_decode_kernel<DK, DV, 4>,
                                                           cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)
                                    : cudaFuncSetAttribute(gdn::mixer_decode_kernel<DK, DV, 8>,
                                                           cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "mixer_decode_kernel smem: %s", cudaGetErrorString(e));
        gdn::LaunchScope timed(st, "mixer_decode_kernel");
        if (args.W <= 4) gdn::mixer_decode_kernel<DK, DV, 4><<<(unsigned)(B * args.H), Sh::THREADS, bytes, st>>>(args);
        else gdn::mixer_decode_kernel<DK, DV, 8><<<(unsigned)(B * args.H), Sh::THREADS, bytes, st>>>(args);
        return launched("mixer_decode_kernel");
    }
};

template <int DK, int DV>
struct RecurrentLaunch {
    static gdn_status_t run(const void* q, const void* k, const void* v, const float* g, const float* beta,
                            const float* S0, const int32_t* cu, int num_seqs, int N, int H, float scale,
                            int in_dt, int y_dt, void* y, float* S_T, cudaStream_t st) {
        using Sh = gdn::RecShape<DK, DV>;
        const unsigned grid = (unsigned)((long long)num_seqs * H * (DV / Sh::SLAB));  // <= 2^31 (host check)
        gdn::LaunchScope timed(st, "recurrent_fwd_kernel");
        gdn::recurrent_fwd_kernel<DK, DV><<<grid, Sh::THREADS, 0, st>>>(
            q, k, v, g, beta, S0, cu, num_seqs, N, H, scale, in_dt, y_dt, y, S_T);
        return launched("recurrent_fwd_kernel");
    }
};

template <int DK, int DV>
struct BwdLaunch {
    static gdn_status_t run(const void* q, const void* k, const void* v, const float* g, const float* beta,
                            const float* S0, const int32_t* cu, int num_seqs, int N, int H, float scale, int in_dt,
                            const void* dy, int dy_dt, const float* dS_T, float* ckpt, float* dq, float* dk, float* dv,
                            float* dg, float* dbeta, float* dS0, cudaStream_t st) {
        using Sh = gdn::RecShape<DK, DV>;
        using Bw = gdn::BwdShape<DK, DV>;
        const unsigned grid = (unsigned)((long long)num_seqs * H * (DV / Sh::SLAB));  // <= 2^31 (host check)
        if (N > 0) {
            const size_t nbytes = (size_t)N * H * DK * 4;
            cudaError_t e = cudaMemsetAsync(dq, 0, nbytes, st);
            if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, nbytes, st);
            if (e == cudaSuccess) e = cudaMemsetAsync(dg, 0, (size_t)N * H * 4, st);
            if (e == cudaSuccess) e = cudaMemsetAsync(dbeta, 0, (size_t)N * H * 4, st);
            if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
            gdn::LaunchScope timed(st, "recurrent_fwd_kernel");
            gdn::recurrent_fwd_kernel<DK, DV><<<grid, Sh::THREADS, 0, st>>>(q, k, v, g, beta, S0, cu, num_seqs, N, H,
                                                                            scale, in_dt, in_dt, nullptr, nullptr,
                                                                            ckpt);
            gdn_status_t r = launched("recurrent_fwd_kernel");
            if (r != GDN_OK) return r;
        }
        cudaError_t e = cudaFuncSetAttribute(gdn::recurrent_bwd_kernel<DK, DV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, Bw::BYTES);
        if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "recurrent_bwd_kernel attribute: %s", cudaGetErrorString(e));
        gdn::LaunchScope timed(st, "recurrent_bwd_kernel");
        gdn::recurrent_bwd_kernel<DK, DV><<<grid, Bw::THREADS, Bw::BYTES, st>>>(
            q, k, v, g, beta, cu, num_seqs, N, H, scale, in_dt, dy, dy_dt, dS_T, ckpt, dq, dk, dv, dg, dbeta, dS0);
        return launched("recurrent_bwd_kernel");
    }
};

template <int DK, int DV>
struct PrepLaunch {
    template <int TAPS>
    static gdn_status_t go(const gdn::PrepMaps& maps, const float* wq, const float* wk, const float* wv, int W,
                           const void* bl, const void* al, const float* A, const float* ba, const int32_t* cu,
                           int num_seqs, int N, int H, float eps, int in_dt, int out_dt, void* q, void* k, void* v,
                           float* g, float* beta, cudaStream_t st) {
        const int esz = in_dt == GDN_F32 ? 4 : 2;
        const int bytes = 2 * gdn::prep_tile_bytes(DK, TAPS, esz) + gdn::prep_tile_bytes(DV, TAPS, esz) + 16 + 128;
        cudaError_t e = cudaFuncSetAttribute(gdn::prep_kernel<DK, DV, TAPS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             bytes);
        if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "prep_kernel smem: %s", cudaGetErrorString(e));
        const unsigned grid = (unsigned)((N + gdn::kPrepRun - 1) / gdn::kPrepRun) * (unsigned)H;
        gdn::LaunchScope timed(st, "prep_kernel");
        gdn::prep_kernel<DK, DV, TAPS><<<grid, gdn::kPrepThreads, bytes, st>>>(maps, wq, wk, wv, W, bl, al, A, ba, cu, num_seqs, N,
                                                                  H, eps, in_dt, out_dt, q, k, v, g, beta,
                                                                  wait_budget());
        return launched("prep_kernel");
    }
    static gdn_status_t run(const void* xq, const void* xk, const void* xv, const float* wq, const float* wk,
                            const float* wv, int W, const void* bl, const void* al, const float* A,
                            const float* ba, const int32_t* cu, int num_seqs, int N, int H, float eps,
                            int in_dt, int out_dt, void* q, void* k, void* v, float* g, float* beta,
                            cudaStream_t st) {
        const int taps = W <= 4 ? 4 : 8;
        const uint32_t rows = (uint32_t)(gdn::kPrepRun + taps - 1);
        gdn::PrepMaps maps;
        if (!gdn::encode_map_3d(&maps.q, xq, in_dt, N, H, DK, DK, rows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !gdn::encode_map_3d(&maps.k, xk, in_dt, N, H, DK, DK, rows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !gdn::encode_map_3d(&maps.v, xv, in_dt, N, H, DV, DV, rows, CU_TENSOR_MAP_SWIZZLE_NONE))
            return fail(GDN_ERR_CUDA, "prep: cuTensorMapEncodeTiled failed");
        if (taps == 4)
            return go<4>(maps, wq, wk, wv, W, bl, al, A, ba, cu, num_seqs, N, H, eps, in_dt, out_dt, q, k, v, g, beta, st);
        return go<8>(maps, wq, wk, wv, W, bl, al, A, ba, cu, num_seqs, N, H, eps, in_dt, out_dt, q, k, v, g, beta, st);
    }
};

// Scratch of gdn_chunk_fwd_noalloc: part of the device image, one copy per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

// The array's device address belongs to the CUDA context that loaded the library's module:
// a reset of the device's primary context unloads the module, and the next context may load
// it elsewhere.  So the address is cached per context, keyed by the context's unique id.
struct NoallocEntry {
    unsigned long long ctx_id;
    void* addr;
};
std::mutex g_noalloc_mu;
std::vector<NoallocEntry> g_noalloc_cache;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<F>(p);
}

// Device address of the scratch array in the calling thread's current context; looked up
// (cudaGetSymbolAddress) the first time a context is seen.
gdn_status_t noalloc_scratch(void** out) {
    static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return fail(GDN_ERR_CUDA, "driver entry points cuCtxGetCurrent / cuCtxGetId");
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return fail(GDN_ERR_CUDA, "cuCtxGetCurrent failed");
    void* p = nullptr;
    if (ctx == nullptr) {  // no context bound to this thread yet: the runtime binds the device's own
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            return fail(GDN_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return fail(GDN_ERR_CUDA, "no current CUDA context");
    }
    unsigned long long id = 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return fail(GDN_ERR_CUDA, "cuCtxGetId failed");
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    for (const NoallocEntry& en : g_noalloc_cache)
        if (en.ctx_id == id) {
            *out = en.addr;
            return GDN_OK;
        }
    if (p == nullptr) {
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            return fail(GDN_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    }
    g_noalloc_cache.push_back({id, p});
    *out = p;
    return GDN_OK;
}

}  // namespace

namespace {

template <int DV, int YT, int ZT>
void launch_out_gate_t(const void* y, const void* z, const float* w, float eps, long long rows, void* out,
                       cudaStream_t st) {
    const long long per_block = (long long)gdn::kGateWarps * gdn::GateShape<DV, YT, ZT>::ROWS_PER_WARP;
    const unsigned grid = (unsigned)((rows + per_block - 1) / per_block);
    gdn::out_gate_kernel<DV, YT, ZT><<<grid, 32 * gdn::kGateWarps, 0, st>>>(y, z, w, eps, rows, out);
}

template <int DV, int YT>
void launch_out_gate_y(const void* y, const void* z, const float* w, float eps, long long rows, int zt, void* out,
                       cudaStream_t st) {
    if (zt == gdn::kF32) launch_out_gate_t<DV, YT, gdn::kF32>(y, z, w, eps, rows, out, st);
    else if (zt == gdn::kBF16) launch_out_gate_t<DV, YT, gdn::kBF16>(y, z, w, eps, rows, out, st);
    else launch_out_gate_t<DV, YT, gdn::kF16>(y, z, w, eps, rows, out, st);
}

template <int DV>
void launch_out_gate(const void* y, const void* z, const float* w, float eps, long long rows, int yt, int zt,
                     void* out, cudaStream_t st) {
    if (yt == gdn::kF32) launch_out_gate_y<DV, gdn::kF32>(y, z, w, eps, rows, zt, out, st);
    else if (yt == gdn::kBF16) launch_out_gate_y<DV, gdn::kBF16>(y, z, w, eps, rows, zt, out, st);
    else launch_out_gate_y<DV, gdn::kF16>(y, z, w, eps, rows, zt, out, st);
}

}  // namespace

namespace {

template <bool BF, int TAPS>
gdn_status_t inproj_go(const gdn::InprojMaps& maps, const gdn::InprojArgs& a, cudaStream_t st) {
    using Cf = gdn::IpCfg<TAPS>;
    const int bytes = Cf::BYTES + Cf::ALIGN;
    cudaError_t e = cudaFuncSetAttribute(gdn::inproj_prep_kernel<BF, TAPS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         bytes);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "inproj_prep_kernel smem: %s", cudaGetErrorString(e));
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "SM count: %s", cudaGetErrorString(e));
    const long long grid = a.n_tiles < sms ? a.n_tiles : sms;  // persistent: one CTA per SM
    gdn::LaunchScope timed(st, "inproj_prep_kernel");
    gdn::inproj_prep_kernel<BF, TAPS><<<(unsigned)grid, Cf::THREADS, bytes, st>>>(maps, a);
    return launched("inproj_prep_kernel");
}

}  // namespace

extern "C" {

int gdn_version(void) { return 100; }

int gdn_bounds_checked(void) {
#ifdef GDN_BOUNDS_CHECK
    return 1;
#else
    return 0;
#endif
}

const char* gdn_status_string(gdn_status_t s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    }
    return "GDN_ERR_UNKNOWN";
}

const char* gdn_last_error_message(void) { return g_msg; }

void gdn_set_wait_budget(uint64_t cycles) { g_wait_budget.store(cycles, std::memory_order_relaxed); }

gdn_status_t gdn_check_device_error(gdn_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
    unsigned word = 0;
    e = cudaMemcpyFromSymbol(&word, gdn::g_error_word, sizeof(word));
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "error word: %s", cudaGetErrorString(e));
    if (word) {
        const unsigned zero = 0;
        cudaMemcpyToSymbol(gdn::g_error_word, &zero, sizeof(zero));
        if (word & gdn::kErrTimeout) return fail(GDN_ERR_TIMEOUT, "a device-side wait ran out (word 0x%x)", word);
        if (word & gdn::kErrSeqlens) return fail(GDN_ERR_INVALID_ARG, "cu_seqlens out of order or range (word 0x%x)", word);
        if (word & gdn::kErrSlot) return fail(GDN_ERR_INVALID_ARG, "state_slot out of range (word 0x%x)", word);
        if (word & gdn::kErrBounds)
            return fail(GDN_ERR_INVALID_ARG, "a device-side bounds check failed: an index outside its tensor (word 0x%x)", word);
        return fail(GDN_ERR_CUDA, "device error word 0x%x", word);
    }
    g_msg[0] = 0;
    return GDN_OK;
}

gdn_status_t gdn_decode_step(const void* q, const void* k, const void* v, const float* g, const float* beta,
                             float* state, const int32_t* state_slot, int num_slots, int B, int H, int dk,
                             int dv, float scale, gdn_dtype_t in_dtype, gdn_dtype_t y_dtype, void* y,
                             gdn_stream_t stream) {
    REQUIRE(B >= 0 && H >= 1 && num_slots >= 0, "bad sizes B=%d H=%d num_slots=%d", B, H, num_slots);
    REQUIRE(head_dim_ok(dk) && head_dim_ok(dv), "dk=%d dv=%d not in {16,32,64,128}", dk, dv);
    REQUIRE(dtype_ok(in_dtype) && dtype_ok(y_dtype), "bad dtype");
    REQUIRE(state_slot != nullptr || num_slots >= B, "num_slots=%d < B=%d without state_slot", num_slots, B);
    REQUIRE((long long)B * H <= 0x7fffffffLL, "B*H too large");
    if (B == 0) return GDN_OK;
    REQUIRE_PTR(q, "q"); REQUIRE_PTR(k, "k"); REQUIRE_PTR(v, "v"); REQUIRE_PTR(g, "g");
    REQUIRE_PTR(beta, "beta"); REQUIRE_PTR(state, "state"); REQUIRE_PTR(y, "y"); OPT_PTR(state_slot, "state_slot");
    return dispatch_dims<DecodeLaunch>(dk, dv, q, k, v, g, beta, state, state_slot, num_slots, B, H, scale,
                                       (int)in_dtype, (int)y_dtype, y, reinterpret_cast<cudaStream_t>(stream));
}

gdn_status_t gdn_mixer_decode_step(const void* x_q, const void* x_k, const void* x_v, const float* conv_w_q,
                                   const float* conv_w_k, const float* conv_w_v, int conv_width,
                                   const void* beta_logit, const void* alpha_logit, const float* A_log,
                                   const float* alpha_bias, const void* z, const float* norm_w, float l2_eps,
                                   float rms_eps, void* conv_state, float* state, const int32_t* state_slot,
                                   int num_slots, int B, int H, int dk, int dv, float scale, gdn_dtype_t in_dtype,
                                   gdn_dtype_t out_dtype, void* out, gdn_stream_t stream) {
    REQUIRE(B >= 0 && H >= 1 && num_slots >= 0, "bad sizes B=%d H=%d num_slots=%d", B, H, num_slots);
    REQUIRE(head_dim_ok(dk) && head_dim_ok(dv), "dk=%d dv=%d not in {16,32,64,128}", dk, dv);
    REQUIRE(dtype_ok(in_dtype) && dtype_ok(out_dtype), "bad dtype");
    REQUIRE(conv_width >= 1 && conv_width <= 8, "conv_width=%d not in [1, 8]", conv_width);
    REQUIRE(l2_eps >= 0.f && rms_eps >= 0.f, "eps < 0");
    REQUIRE(state_slot != nullptr || num_slots >= B, "num_slots=%d < B=%d without state_slot", num_slots, B);
    REQUIRE((long long)B * H <= 0x7fffffffLL, "B*H too large");
    if (B == 0) return GDN_OK;
    REQUIRE_PTR(x_q, "x_q"); REQUIRE_PTR(x_k, "x_k"); REQUIRE_PTR(x_v, "x_v");
    REQUIRE_PTR(conv_w_q, "conv_w_q"); REQUIRE_PTR(conv_w_k, "conv_w_k"); REQUIRE_PTR(conv_w_v, "conv_w_v");
    REQUIRE_PTR(beta_logit, "beta_logit"); REQUIRE_PTR(alpha_logit, "alpha_logit");
    REQUIRE_PTR(A_log, "A_log"); REQUIRE_PTR(alpha_bias, "alpha_bias"); REQUIRE_PTR(z, "z");
    REQUIRE_PTR(norm_w, "norm_w"); REQUIRE_PTR(state, "state"); REQUIRE_PTR(out, "out");
    if (conv_width > 1) REQUIRE_PTR(conv_state, "conv_state");
    OPT_PTR(state_slot, "state_slot");
    const gdn::MixerDecodeArgs args{x_q, x_k, x_v, conv_w_q, conv_w_k, conv_w_v, conv_width, beta_logit,
                                    alpha_logit, A_log, alpha_bias, z, norm_w, l2_eps, rms_eps, conv_state,
                                    state, state_slot, num_slots, H, scale, (int)in_dtype, (int)out_dtype, out,
                                    wait_budget()};
    return dispatch_dims<MixerDecodeLaunch>(dk, dv, args, B, reinterpret_cast<cudaStream_t>(stream));
}

size_t gdn_chunk_fwd_workspace_size(int N, int num_seqs, int H, int dk, int dv, int chunk) {
    return gdn::chunk_tc_workspace_bytes(N, num_seqs, H, dk, dv, chunk);
}

gdn_status_t gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           const float* S0, const int32_t* cu_seqlens, int num_seqs, int N, int H, int dk,
                           int dv, int chunk, float scale, gdn_dtype_t in_dtype, gdn_dtype_t y_dtype, void* y,
                           float* S_T, void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    REQUIRE(N >= 0 && H >= 1 && num_seqs >= 1, "bad sizes N=%d H=%d num_seqs=%d", N, H, num_seqs);
    REQUIRE(head_dim_ok(dk) && head_dim_ok(dv), "dk=%d dv=%d not in {16,32,64,128}", dk, dv);
    REQUIRE(dtype_ok(in_dtype) && dtype_ok(y_dtype), "bad dtype");
    REQUIRE(chunk >= 0, "chunk=%d < 0", chunk);
    REQUIRE(cu_seqlens != nullptr || N % num_seqs == 0, "N=%d not a multiple of num_seqs=%d", N, num_seqs);
    REQUIRE((long long)N * H * (dk > dv ? dk : dv) < (1LL << 40), "problem too large");
    REQUIRE((long long)num_seqs * H * 128 <= 0x7fffffffLL, "num_seqs*H too large (%d x %d)", num_seqs, H);
    if (N == 0 && S_T == nullptr) return GDN_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (chunk != 0 && chunk != 64)
        return fail(GDN_ERR_UNSUPPORTED, "chunk=%d: the tensor-core path is built for chunk 64 (chunk 0 for the recurrence)", chunk);
    if (chunk == 64 && (dk != 128 || dv != 128 || in_dtype == GDN_F32))
        return fail(GDN_ERR_UNSUPPORTED, "chunked path needs dk=dv=128 and bf16/f16 inputs (use chunk=0)");
    OPT_PTR(S0, "S0"); OPT_PTR(S_T, "S_T"); OPT_PTR(cu_seqlens, "cu_seqlens");
    if (N == 0)  // every sequence is empty: S_T = S0 (or zero), by the recurrence, which reads no token
        return dispatch_dims<RecurrentLaunch>(dk, dv, q, k, v, g, beta, S0, cu_seqlens, num_seqs, N, H, scale,
                                              (int)in_dtype, (int)y_dtype, y, S_T, st);
    REQUIRE_PTR(g, "g"); REQUIRE_PTR(beta, "beta"); REQUIRE_PTR(q, "q"); REQUIRE_PTR(k, "k");
    REQUIRE_PTR(v, "v"); REQUIRE_PTR(y, "y");
    OPT_PTR(workspace, "workspace");
    if (chunk == 0)
        return dispatch_dims<RecurrentLaunch>(dk, dv, q, k, v, g, beta, S0, cu_seqlens, num_seqs, N, H, scale,
                                              (int)in_dtype, (int)y_dtype, y, S_T, st);
    const size_t need = gdn::chunk_tc_workspace_bytes(N, num_seqs, H, dk, dv, chunk);
    REQUIRE(workspace_bytes >= need && (need == 0 || workspace != nullptr), "workspace of %zu bytes < %zu",
            workspace_bytes, need);
    gdn::ChunkArgs a{q, k, v, g, beta, S0, cu_seqlens, num_seqs, N, H, chunk, scale, (int)in_dtype,
                     (int)y_dtype, y, S_T, workspace, wait_budget()};
    const char* why = nullptr;
    cudaError_t e = gdn::chunk_tc_launch(a, st, &why);
    if (why) return fail(GDN_ERR_CUDA, "chunk_tc: %s", why);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "chunk_tc: %s", cudaGetErrorString(e));
    return GDN_OK;
}

size_t gdn_chunk_fwd_prep_workspace_size(int N, int num_seqs, int H, int dk, int dv, int chunk) {
    return gdn::chunk_tc_workspace_bytes(N, num_seqs, H, dk, dv, chunk);
}

gdn_status_t gdn_chunk_fwd_prep(const void* x_q, const void* x_k, const void* x_v, const float* conv_w_q,
                                const float* conv_w_k, const float* conv_w_v, int conv_width, const void* beta_logit,
                                const void* alpha_logit, const float* A_log, const float* alpha_bias, float l2_eps,
                                const float* S0, const int32_t* cu_seqlens, int num_seqs, int N, int H, int dk,
                                int dv, int chunk, float scale, gdn_dtype_t in_dtype, gdn_dtype_t qkv_dtype,
                                gdn_dtype_t y_dtype, void* y, float* S_T, void* workspace, size_t workspace_bytes,
                                gdn_stream_t stream) {
    REQUIRE(N >= 0 && H >= 1 && num_seqs >= 1, "bad sizes N=%d H=%d num_seqs=%d", N, H, num_seqs);
    REQUIRE(head_dim_ok(dk) && head_dim_ok(dv), "dk=%d dv=%d not in {16,32,64,128}", dk, dv);
    REQUIRE(dtype_ok(in_dtype) && dtype_ok(qkv_dtype) && dtype_ok(y_dtype), "bad dtype");
    REQUIRE(conv_width >= 1 && conv_width <= 8, "conv_width=%d not in [1, 8]", conv_width);
    REQUIRE(l2_eps >= 0.f, "l2_eps < 0");
    REQUIRE(cu_seqlens != nullptr || N % num_seqs == 0, "N=%d not a multiple of num_seqs=%d", N, num_seqs);
    REQUIRE((long long)N * H * 128 < (1LL << 40), "problem too large");
    REQUIRE((long long)num_seqs * H * 128 <= 0x7fffffffLL, "num_seqs*H too large (%d x %d)", num_seqs, H);
    if (chunk != 64 || dk != 128 || dv != 128 || in_dtype == GDN_F32 || qkv_dtype == GDN_F32)
        return fail(GDN_ERR_UNSUPPORTED, "the fused prep runs the tensor-core path only (chunk 64, dk=dv=128, "
                                         "16-bit inputs and q/k/v format)");
    if (N == 0)  // every sequence is empty: S_T = S0 (or zero)
        return gdn_chunk_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, S0, cu_seqlens, num_seqs, 0, H, dk, dv, 0,
                             scale, qkv_dtype, y_dtype, y, S_T, nullptr, 0, stream);
    REQUIRE_PTR(x_q, "x_q"); REQUIRE_PTR(x_k, "x_k"); REQUIRE_PTR(x_v, "x_v");
    REQUIRE_PTR(conv_w_q, "conv_w_q"); REQUIRE_PTR(conv_w_k, "conv_w_k"); REQUIRE_PTR(conv_w_v, "conv_w_v");
    REQUIRE_PTR(beta_logit, "beta_logit"); REQUIRE_PTR(alpha_logit, "alpha_logit");
    REQUIRE_PTR(A_log, "A_log"); REQUIRE_PTR(alpha_bias, "alpha_bias"); REQUIRE_PTR(y, "y");
    OPT_PTR(S0, "S0"); OPT_PTR(S_T, "S_T"); OPT_PTR(cu_seqlens, "cu_seqlens");
    const size_t need = gdn_chunk_fwd_prep_workspace_size(N, num_seqs, H, dk, dv, chunk);
    REQUIRE_PTR(workspace, "workspace");
    REQUIRE(workspace_bytes >= need, "workspace of %zu bytes < %zu", workspace_bytes, need);
    gdn::PrepIn p{conv_w_q, conv_w_k, conv_w_v, conv_width, beta_logit, alpha_logit, A_log, alpha_bias, l2_eps,
                  (int)in_dtype};
    gdn::ChunkArgs a{nullptr, nullptr, nullptr, nullptr, nullptr, S0, cu_seqlens, num_seqs, N, H, chunk, scale,
                     (int)qkv_dtype, (int)y_dtype, y, S_T, workspace, wait_budget()};
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const char* why = nullptr;
    cudaError_t e = gdn::chunk_tc_prep_launch(a, p, x_q, x_k, x_v, st, &why);
    if (why) return fail(GDN_ERR_CUDA, "chunk_tc: %s", why);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "chunk_tc: %s", cudaGetErrorString(e));
    return GDN_OK;
}

size_t gdn_chunk_bwd_workspace_size(int N, int num_seqs, int H, int dk, int dv) {
    if (N <= 0 || num_seqs <= 0 || H <= 0 || dk <= 0 || dv <= 0) return 0;
    return (size_t)gdn::bwd_block_bound(N, num_seqs) * H * dk * dv * 4;
}

gdn_status_t gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           const float* S0, const int32_t* cu_seqlens, int num_seqs, int N, int H, int dk, int dv,
                           float scale, gdn_dtype_t in_dtype, const void* dy, gdn_dtype_t dy_dtype, const float* dS_T,
                           float* dq, float* dk_out, float* dv_out, float* dg, float* dbeta, float* dS0,
                           void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    REQUIRE(N >= 0 && H >= 1 && num_seqs >= 1, "bad sizes N=%d H=%d num_seqs=%d", N, H, num_seqs);
    REQUIRE(head_dim_ok(dk) && head_dim_ok(dv), "dk=%d dv=%d not in {16,32,64,128}", dk, dv);
    REQUIRE(dtype_ok(in_dtype) && dtype_ok(dy_dtype), "bad dtype");
    REQUIRE(cu_seqlens != nullptr || N % num_seqs == 0, "N=%d not a multiple of num_seqs=%d", N, num_seqs);
    REQUIRE((long long)N * H * (dk > dv ? dk : dv) < (1LL << 40), "problem too large");
    REQUIRE((long long)num_seqs * H * 128 <= 0x7fffffffLL, "num_seqs*H too large (%d x %d)", num_seqs, H);
    OPT_PTR(S0, "S0"); OPT_PTR(dS_T, "dS_T"); OPT_PTR(cu_seqlens, "cu_seqlens");
    REQUIRE_PTR(dS0, "dS0");
    if (N > 0) {
        REQUIRE_PTR(q, "q"); REQUIRE_PTR(k, "k"); REQUIRE_PTR(v, "v"); REQUIRE_PTR(g, "g"); REQUIRE_PTR(beta, "beta");
        REQUIRE_PTR(dy, "dy"); REQUIRE_PTR(dq, "dq"); REQUIRE_PTR(dk_out, "dk"); REQUIRE_PTR(dv_out, "dv");
        REQUIRE_PTR(dg, "dg"); REQUIRE_PTR(dbeta, "dbeta");
        const size_t need = gdn_chunk_bwd_workspace_size(N, num_seqs, H, dk, dv);
        REQUIRE_PTR(workspace, "workspace");
        REQUIRE(workspace_bytes >= need, "workspace of %zu bytes < %zu", workspace_bytes, need);
    }
    return dispatch_dims<BwdLaunch>(dk, dv, q, k, v, g, beta, S0, cu_seqlens, num_seqs, N, H, scale, (int)in_dtype, dy,
                                    (int)dy_dtype, dS_T, reinterpret_cast<float*>(workspace), dq, dk_out, dv_out, dg,
                                    dbeta, dS0, reinterpret_cast<cudaStream_t>(stream));
}

gdn_status_t gdn_chunk_fwd_gated(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                 const float* S0, const int32_t* cu_seqlens, int num_seqs, int N, int H, int dk,
                                 int dv, int chunk, float scale, gdn_dtype_t in_dtype, const void* z,
                                 const float* norm_w, float eps, gdn_dtype_t io_dtype, void* out, float* S_T,
                                 void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
    REQUIRE(N >= 0 && H >= 1 && num_seqs >= 1, "bad sizes N=%d H=%d num_seqs=%d", N, H, num_seqs);
    REQUIRE(dtype_ok(in_dtype) && dtype_ok(io_dtype), "bad dtype");
    REQUIRE(eps >= 0.f, "eps < 0");
    REQUIRE(cu_seqlens != nullptr || N % num_seqs == 0, "N=%d not a multiple of num_seqs=%d", N, num_seqs);
    REQUIRE((long long)N * H * 128 < (1LL << 40), "problem too large");
    REQUIRE((long long)num_seqs * H * 128 <= 0x7fffffffLL, "num_seqs*H too large (%d x %d)", num_seqs, H);
    if (chunk != 64 || dk != 128 || dv != 128 || in_dtype == GDN_F32 || io_dtype == GDN_F32)
        return fail(GDN_ERR_UNSUPPORTED, "the gated variant runs the tensor-core path only (chunk 64, dk=dv=128, "
                                         "bf16/f16 inputs, bf16/f16 z and out)");
    if (N == 0 && S_T == nullptr) return GDN_OK;
    OPT_PTR(S0, "S0"); OPT_PTR(S_T, "S_T"); OPT_PTR(cu_seqlens, "cu_seqlens");
    if (N == 0)  // every sequence is empty: S_T = S0 (or zero), by the recurrence, which reads no token
        return dispatch_dims<RecurrentLaunch>(dk, dv, q, k, v, g, beta, S0, cu_seqlens, num_seqs, N, H, scale,
                                              (int)in_dtype, (int)io_dtype, nullptr, S_T,
                                              reinterpret_cast<cudaStream_t>(stream));
    REQUIRE_PTR(g, "g"); REQUIRE_PTR(beta, "beta"); REQUIRE_PTR(q, "q"); REQUIRE_PTR(k, "k");
    REQUIRE_PTR(v, "v"); REQUIRE_PTR(z, "z"); REQUIRE_PTR(norm_w, "norm_w"); REQUIRE_PTR(out, "out");
    OPT_PTR(workspace, "workspace");
    const size_t need = gdn::chunk_tc_workspace_bytes(N, num_seqs, H, dk, dv, chunk);
    REQUIRE(workspace_bytes >= need && (need == 0 || workspace != nullptr), "workspace of %zu bytes < %zu",
            workspace_bytes, need);
    gdn::ChunkArgs a{q, k, v, g, beta, S0, cu_seqlens, num_seqs, N, H, chunk, scale, (int)in_dtype,
                     (int)io_dtype, nullptr, S_T, workspace, wait_budget(), z, norm_w, eps, (int)io_dtype, out};
    const char* why = nullptr;
    cudaError_t e = gdn::chunk_tc_launch(a, reinterpret_cast<cudaStream_t>(stream), &why);
    if (why) return fail(GDN_ERR_CUDA, "chunk_tc: %s", why);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "chunk_tc gated: %s", cudaGetErrorString(e));
    return GDN_OK;
}

gdn_status_t gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                   const float* S0, const int32_t* cu_seqlens, int num_seqs, int N, int H, int dk,
                                   int dv, int chunk, float scale, gdn_dtype_t in_dtype, gdn_dtype_t y_dtype, void* y,
                                   float* S_T, gdn_stream_t stream) {
    // only a call the tensor-core path accepts needs scratch; anything else goes straight to
    // gdn_chunk_fwd's own checks, so both entry points answer a bad call the same way
    const bool tc = chunk == 64 && dk == 128 && dv == 128 && in_dtype != GDN_F32;
    const size_t need = tc ? gdn::chunk_tc_workspace_bytes(N, num_seqs, H, dk, dv, chunk) : 0;
    if (need > GDN_NOALLOC_SCRATCH_BYTES)
        return fail(GDN_ERR_INVALID_ARG, "needs %zu bytes of scratch; the no-allocation entry point holds %llu",
                    need, (unsigned long long)GDN_NOALLOC_SCRATCH_BYTES);
    void* ws = nullptr;
    if (need > 0) {
        const gdn_status_t st = noalloc_scratch(&ws);
        if (st != GDN_OK) return st;
    }
    return gdn_chunk_fwd(q, k, v, g, beta, S0, cu_seqlens, num_seqs, N, H, dk, dv, chunk, scale, in_dtype, y_dtype, y,
                         S_T, ws, need, stream);
}

gdn_status_t gdn_prep(const void* x_q, const void* x_k, const void* x_v, const float* conv_w_q,
                      const float* conv_w_k, const float* conv_w_v, int conv_width, const void* beta_logit,
                      const void* alpha_logit, const float* A_log, const float* alpha_bias,
                      const int32_t* cu_seqlens, int num_seqs, int N, int H, int dk, int dv, float l2_eps,
                      gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* q, void* k, void* v, float* g_out,
                      float* beta_out, gdn_stream_t stream) {
    REQUIRE(N >= 0 && H >= 1 && num_seqs >= 1, "bad sizes N=%d H=%d num_seqs=%d", N, H, num_seqs);
    REQUIRE(head_dim_ok(dk) && head_dim_ok(dv), "dk=%d dv=%d not in {16,32,64,128}", dk, dv);
    REQUIRE(dtype_ok(in_dtype) && dtype_ok(out_dtype), "bad dtype");
    REQUIRE(conv_width >= 1 && conv_width <= 8, "conv_width=%d not in [1, 8]", conv_width);
    REQUIRE(cu_seqlens != nullptr || N % num_seqs == 0, "N=%d not a multiple of num_seqs=%d", N, num_seqs);
    REQUIRE(l2_eps >= 0.f, "l2_eps < 0");
    if (N == 0) return GDN_OK;
    REQUIRE_PTR(x_q, "x_q"); REQUIRE_PTR(x_k, "x_k"); REQUIRE_PTR(x_v, "x_v");
    REQUIRE_PTR(conv_w_q, "conv_w_q"); REQUIRE_PTR(conv_w_k, "conv_w_k"); REQUIRE_PTR(conv_w_v, "conv_w_v");
    REQUIRE_PTR(beta_logit, "beta_logit"); REQUIRE_PTR(alpha_logit, "alpha_logit");
    REQUIRE_PTR(A_log, "A_log"); REQUIRE_PTR(alpha_bias, "alpha_bias");
    REQUIRE_PTR(q, "q"); REQUIRE_PTR(k, "k"); REQUIRE_PTR(v, "v"); REQUIRE_PTR(g_out, "g_out");
    REQUIRE_PTR(beta_out, "beta_out"); OPT_PTR(cu_seqlens, "cu_seqlens");
    return dispatch_dims<PrepLaunch>(dk, dv, x_q, x_k, x_v, conv_w_q, conv_w_k, conv_w_v, conv_width, beta_logit,
                                     alpha_logit, A_log, alpha_bias, cu_seqlens, num_seqs, N, H, l2_eps,
                                     (int)in_dtype, (int)out_dtype, q, k, v, g_out, beta_out,
                                     reinterpret_cast<cudaStream_t>(stream));
}

gdn_status_t gdn_inproj_prep(const void* x, const void* w, int D, const float* conv_w_q, const float* conv_w_k,
                             const float* conv_w_v, int conv_width, const float* A_log, const float* alpha_bias,
                             const int32_t* cu_seqlens, int num_seqs, int N, int H, int dk, int dv, float l2_eps,
                             gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* q, void* k, void* v, void* z,
                             float* g_out, float* beta_out, gdn_stream_t stream) {
    REQUIRE(N >= 0 && H >= 1 && num_seqs >= 1, "bad sizes N=%d H=%d num_seqs=%d", N, H, num_seqs);
    REQUIRE(dtype_ok(in_dtype) && dtype_ok(out_dtype), "bad dtype");
    REQUIRE(conv_width >= 1 && conv_width <= 8, "conv_width=%d not in [1, 8]", conv_width);
    REQUIRE(cu_seqlens != nullptr || N % num_seqs == 0, "N=%d not a multiple of num_seqs=%d", N, num_seqs);
    REQUIRE(l2_eps >= 0.f, "l2_eps < 0");
    REQUIRE(D >= 64 && D % 64 == 0, "D=%d not a positive multiple of 64", D);
    if (dk != 128 || dv != 128 || H % 16 != 0 || H > 128 || in_dtype == GDN_F32 || out_dtype == GDN_F32)
        return fail(GDN_ERR_UNSUPPORTED,
                    "gdn_inproj_prep is built for dk = dv = 128, H a multiple of 16 up to 128 and 16-bit x, w and "
                    "outputs (dk=%d dv=%d H=%d)", dk, dv, H);
    REQUIRE((long long)N * D < (1LL << 40), "N * D too large");
    if (N == 0) return GDN_OK;
    REQUIRE_PTR(x, "x"); REQUIRE_PTR(w, "w");
    REQUIRE_PTR(conv_w_q, "conv_w_q"); REQUIRE_PTR(conv_w_k, "conv_w_k"); REQUIRE_PTR(conv_w_v, "conv_w_v");
    REQUIRE_PTR(A_log, "A_log"); REQUIRE_PTR(alpha_bias, "alpha_bias");
    REQUIRE_PTR(q, "q"); REQUIRE_PTR(k, "k"); REQUIRE_PTR(v, "v"); OPT_PTR(z, "z");
    REQUIRE_PTR(g_out, "g_out"); REQUIRE_PTR(beta_out, "beta_out"); OPT_PTR(cu_seqlens, "cu_seqlens");
    const int taps = conv_width <= 4 ? 4 : 8;
    const int rows_out = 128 - (taps - 1);
    gdn::InprojArgs a;
    a.N = N; a.D = D; a.H = H; a.W = conv_width;
    a.nq = H * 128 / 256;
    a.has_z = z != nullptr;
    a.n_tiles_n = (3 + a.has_z) * a.nq + 1;
    a.n_tiles = (long long)((N + rows_out - 1) / rows_out) * a.n_tiles_n;
    a.conv_q = conv_w_q; a.conv_k = conv_w_k; a.conv_v = conv_w_v;
    a.A_log = A_log; a.alpha_bias = alpha_bias;
    a.cu = cu_seqlens; a.num_seqs = num_seqs; a.eps = l2_eps; a.out_dt = (int)out_dtype;
    a.q = q; a.k = k; a.v = v; a.z = z; a.g = g_out; a.beta = beta_out;
    a.budget = wait_budget();
    const bool bf = in_dtype == GDN_BF16;
    const long long wrows = 4LL * H * 128 + 2 * H;
    gdn::InprojMaps maps;
    if (!gdn::encode_map_2d(&maps.x, x, bf, N, D, 64, 128) || !gdn::encode_map_2d(&maps.w, w, bf, wrows, D, 64, 256) ||
        !gdn::encode_map_2d(&maps.wg, w, bf, wrows, D, 64, (uint32_t)(2 * H)))
        return fail(GDN_ERR_CUDA, "inproj: cuTensorMapEncodeTiled failed");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (bf) return taps == 4 ? inproj_go<true, 4>(maps, a, st) : inproj_go<true, 8>(maps, a, st);
    return taps == 4 ? inproj_go<false, 4>(maps, a, st) : inproj_go<false, 8>(maps, a, st);
}

gdn_status_t gdn_out_gate(const void* y, const void* z, const float* norm_w, float eps, int N, int H, int dv,
                          gdn_dtype_t y_dtype, gdn_dtype_t io_dtype, void* out, gdn_stream_t stream) {
    REQUIRE(N >= 0 && H >= 1, "bad sizes N=%d H=%d", N, H);
    REQUIRE(head_dim_ok(dv), "dv=%d not in {16,32,64,128}", dv);
    REQUIRE(dtype_ok(y_dtype) && dtype_ok(io_dtype), "bad dtype");
    REQUIRE(eps >= 0.f, "eps < 0");
    if (N == 0) return GDN_OK;
    REQUIRE_PTR(y, "y"); REQUIRE_PTR(z, "z"); REQUIRE_PTR(norm_w, "norm_w"); REQUIRE_PTR(out, "out");
    const long long rows = (long long)N * H;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    gdn::LaunchScope timed(st, "out_gate_kernel");
    switch (dv) {
        case 16: launch_out_gate<16>(y, z, norm_w, eps, rows, (int)y_dtype, (int)io_dtype, out, st); break;
        case 32: launch_out_gate<32>(y, z, norm_w, eps, rows, (int)y_dtype, (int)io_dtype, out, st); break;
        case 64: launch_out_gate<64>(y, z, norm_w, eps, rows, (int)y_dtype, (int)io_dtype, out, st); break;
        default: launch_out_gate<128>(y, z, norm_w, eps, rows, (int)y_dtype, (int)io_dtype, out, st); break;
    }
    return launched("out_gate_kernel");
}

gdn_status_t gdn_state_map_apply(const float* M, const float* B, const float* S_in, float* S_out, int rows, int dk,
                                 int dv, gdn_stream_t stream) {
    REQUIRE(rows >= 0, "rows=%d < 0", rows);
    REQUIRE(head_dim_ok(dk) && head_dim_ok(dv), "dk=%d dv=%d not in {16,32,64,128}", dk, dv);
    if (rows == 0) return GDN_OK;
    REQUIRE_PTR(M, "M"); REQUIRE_PTR(S_in, "S_in"); REQUIRE_PTR(S_out, "S_out"); OPT_PTR(B, "B");
    const size_t nm = (size_t)rows * dk * dk * 4, ns = (size_t)rows * dk * dv * 4;
    auto overlap = [](const void* a, size_t na, const void* b, size_t nb) {
        const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
        return x < y + nb && y < x + na;
    };
    REQUIRE(!overlap(S_out, ns, S_in, ns) && !overlap(S_out, ns, M, nm) && (B == nullptr || !overlap(S_out, ns, B, ns)),
            "S_out overlaps an input");
    const long long grid = (long long)rows * (dk / 16) * (dv / 16);
    REQUIRE(grid <= 0x7fffffffLL, "rows=%d too large", rows);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    gdn::LaunchScope timed(st, "state_map_kernel");
    gdn::state_map_kernel<<<(unsigned)grid, 256, 0, st>>>(M, B, S_in, S_out, dk, dv);
    return launched("state_map_kernel");
}

gdn_status_t gdn_timing_start(int max_launches) {
    REQUIRE(max_launches >= 1 && max_launches <= (1 << 20), "max_launches=%d not in [1, 2^20]", max_launches);
    gdn::LaunchTimer& t = gdn::launch_timer();
    std::lock_guard<std::mutex> lock(t.mu);
    REQUIRE(!t.on, "timing is already on");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    t.pool.reserve(2 * (size_t)max_launches);
    for (int i = 0; i < 2 * max_launches; ++i) {
        cudaEvent_t ev = nullptr;
        e = cudaEventCreate(&ev);
        if (e != cudaSuccess) {
            for (cudaEvent_t x : t.pool) cudaEventDestroy(x);
            t.pool.clear();
            return fail(GDN_ERR_CUDA, "cudaEventCreate: %s", cudaGetErrorString(e));
        }
        t.pool.push_back(ev);
    }
    t.names.clear();
    t.device = dev;
    ++t.generation;
    t.on = true;
    return GDN_OK;
}

gdn_status_t gdn_timing_stop(int cap, const char** names, int* launches, double* total_ms, int* n_kernels) {
    REQUIRE(cap >= 0 && (cap == 0 || (names && launches && total_ms)), "bad output arrays (cap=%d)", cap);
    gdn::LaunchTimer& t = gdn::launch_timer();
    std::lock_guard<std::mutex> lock(t.mu);
    REQUIRE(t.on, "timing is not on");
    gdn_status_t status = GDN_OK;
    std::vector<const char*> kn;
    std::vector<int> cnt;
    std::vector<double> ms;
    for (size_t i = 0; i < t.names.size(); ++i) {
        float dt = 0.f;
        cudaError_t e = cudaEventSynchronize(t.pool[2 * i + 1]);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&dt, t.pool[2 * i], t.pool[2 * i + 1]);
        if (e != cudaSuccess) {
            status = fail(GDN_ERR_CUDA, "timing event: %s", cudaGetErrorString(e));
            break;
        }
        size_t j = 0;
        while (j < kn.size() && std::strcmp(kn[j], t.names[i]) != 0) ++j;
        if (j == kn.size()) {
            kn.push_back(t.names[i]);
            cnt.push_back(0);
            ms.push_back(0.0);
        }
        cnt[j] += 1;
        ms[j] += dt;
    }
    for (cudaEvent_t x : t.pool) cudaEventDestroy(x);
    t.pool.clear();
    t.names.clear();
    ++t.generation;
    t.on = false;
    if (status != GDN_OK) return status;
    for (size_t j = 0; j < kn.size() && (int)j < cap; ++j) {
        names[j] = kn[j];
        launches[j] = cnt[j];
        total_ms[j] = ms[j];
    }
    if (n_kernels) *n_kernels = (int)kn.size();
    return GDN_OK;
}

}  // extern "C"
