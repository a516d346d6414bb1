// The C ABI (include/moe.h): argument checks on the host, workspace carving,
// and the launch sequence of the layer on one stream.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <string>

#include <cudaTypedefs.h>

#include "../../include/moe.h"
#include "common.cuh"
#include "internal.h"

namespace {

thread_local std::string g_err;

moe_status fail(moe_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

moe_status cuda_fail(cudaError_t e, const char *where) {
    return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr uint64_t kWaitTimeoutNs = 1000000000ull;  // 1 s per wait

int num_sms_current() {
    static std::atomic<int> cache[64];  // zero-initialised (static storage); any thread may fill an entry
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    if (dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c != 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(moe_dtype dt) { return dt == MOE_BF16 ? 2 : 4; }

bool use_tensor_cores(moe_dtype dt, int d, int d_ff) {
    return dt == MOE_BF16 && d % 8 == 0 && d_ff % 8 == 0;
}

moe_status check_shape(int64_t N, int d, int E, int k, moe_dtype dt) {
    if (dt != MOE_F32 && dt != MOE_BF16) return fail(MOE_ERR_INVALID_ARG, "dtype must be MOE_F32 or MOE_BF16");
    if (N < 0) return fail(MOE_ERR_INVALID_ARG, "N must be >= 0 (got %lld)", (long long)N);
    if (d < 1) return fail(MOE_ERR_INVALID_ARG, "d must be >= 1 (got %d)", d);
    if (E < 1 || E > 256) return fail(MOE_ERR_INVALID_ARG, "E must be in [1, 256] (got %d)", E);
    if (k < 1 || k > E) return fail(MOE_ERR_INVALID_ARG, "k must be in [1, E] (got k=%d, E=%d)", k, E);
    if (N * static_cast<int64_t>(k) > INT32_MAX)
        return fail(MOE_ERR_INVALID_ARG, "N * k must fit in int32 (got %lld)", (long long)(N * k));
    return MOE_OK;
}

#define REQUIRE_PTR(p, name)                                                                    \
    do {                                                                                        \
        if ((p) == nullptr) return fail(MOE_ERR_INVALID_ARG, "%s must not be NULL", name);      \
        if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "%s must be 16-byte aligned", name); \
    } while (0)
#define OPTIONAL_PTR(p, name)                                                                   \
    do {                                                                                        \
        if ((p) != nullptr && !aligned16(p))                                                    \
            return fail(MOE_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);               \
    } while (0)

int64_t rows_for(int64_t N, int E, int k, int64_t C) {
    int64_t r = N * k;
    if (static_cast<int64_t>(E) * C < r) r = static_cast<int64_t>(E) * C;
    return (r + 127) / 128 * 128;
}

size_t ffn_ws_bytes(int64_t rows, int d, int E, int d_ff, moe_dtype dt) {
    if (use_tensor_cores(dt, d, d_ff)) return moe::tc_ffn_ws_bytes(rows, d, d_ff, E, num_sms_current());
    return moe::align_up(static_cast<size_t>(rows) * d_ff * elem_bytes(dt), 256);
}

struct FwdLayout {
    size_t status, topk, gates, slot, counts, offsets, dws, w3, xg, og, ffn, fused, total;
};

// Whether small batches run the whole layer as one cooperative kernel when the
// shape allows (decode_fused.cu).  Off unless MOE_FUSED_DECODE is a nonzero
// number or moe_set_fused_small_batch(1) was called: on a B200 the separate
// decode-plan kernels stream the weights faster.  -1: not read yet.
std::atomic<int> g_fused_small_batch{-1};

bool fused_decode_enabled() {
    int v = g_fused_small_batch.load(std::memory_order_relaxed);
    if (v < 0) {
        const char *e = getenv("MOE_FUSED_DECODE");
        int want = (e != nullptr && atoi(e) != 0) ? 1 : 0;
        int expected = -1;
        g_fused_small_batch.compare_exchange_strong(expected, want);
        v = g_fused_small_batch.load(std::memory_order_relaxed);
    }
    return v != 0;
}

// Whether moe_forward takes the fused small-batch kernel (pointers nullable:
// then their alignment is assumed).
bool use_fused_decode(const void *x, const float *W_g, int64_t N, int d, int E, int d_ff, int k, int64_t rows,
                      moe_dtype dt, int act, const float *b_up, const float *b_down) {
    if (!fused_decode_enabled() || dt != MOE_BF16 || !use_tensor_cores(dt, d, d_ff) || act != MOE_ACT_RELU ||
        b_up != nullptr || b_down != nullptr)
        return false;
    const int sms = num_sms_current();
    const moe::TcPlan p = moe::plan_tc_ffn(rows, d, d_ff, E, sms);
    if (!p.decode || p.splits_up < 2) return false;
    static const uint64_t kAligned[2] = {0, 0};
    const void *xa = x ? x : kAligned;
    const float *wa = W_g ? W_g : reinterpret_cast<const float *>(kAligned);
    return moe::decode_fused_eligible(xa, wa, N, d, E, d_ff, k, rows, sms);
}

FwdLayout forward_layout(int64_t N, int d, int E, int d_ff, int k, int64_t rows, moe_dtype dt) {
    using moe::align_up;
    FwdLayout L{};
    size_t o = 0;
    L.status = o; o += moe::kStatusBytes;
    const size_t nk = static_cast<size_t>(N) * k;
    L.topk = o; o += align_up(nk * 4, 256);
    L.gates = o; o += align_up(nk * 4, 256);
    L.slot = o; o += align_up(nk * 4, 256);
    L.counts = o; o += align_up(static_cast<size_t>(E) * 4, 256);
    L.offsets = o; o += align_up(static_cast<size_t>(E + 1) * 4, 256);
    L.dws = o; o += moe::dispatch_ws_bytes(N, E, k);
    L.w3 = o; o += (dt == MOE_BF16) ? moe::route_tc_w3_bytes(d, E) : 0;  // pre-split router weights
    L.xg = o; o += align_up(static_cast<size_t>(rows) * d * elem_bytes(dt), 256);
    L.og = o; o += align_up(static_cast<size_t>(rows) * d * elem_bytes(dt), 256);
    L.ffn = o; o += ffn_ws_bytes(rows, d, E, d_ff, dt);
    L.fused = o; o += (N <= 64 && dt == MOE_BF16) ? moe::decode_fused_scratch_bytes(N, d, E) : 0;
    L.total = o;
    return L;
}

// H_keep (nullable): the caller's [rows][d_ff] buffer for the hidden
// activations; null keeps them in the workspace.
moe_status run_ffn(const void *xg, const int32_t *offsets, const int32_t *counts, const void *W_up,
                   const void *W_down, moe_dtype dt, int64_t rows, int d, int d_ff, int E, void *out,
                   void *ffn_ws, bool combine_reads_parts, float **parts_out, int *nparts_out,
                   uint32_t *status, cudaStream_t s, int act, const float *b_up, const float *b_down,
                   void *H_keep = nullptr) {
    cudaError_t e;
    if (parts_out) *parts_out = nullptr;
    if (nparts_out) *nparts_out = 0;
    if (use_tensor_cores(dt, d, d_ff)) {
        const int sms = num_sms_current();
        const moe::TcPlan p = moe::plan_tc_ffn(rows, d, d_ff, E, sms);
        uint8_t *w = static_cast<uint8_t *>(ffn_ws);
        void *H = H_keep ? H_keep : w;
        float *parts = p.decode ? reinterpret_cast<float *>(w + moe::align_up(static_cast<size_t>(rows) * d_ff * 2, 256))
                                : nullptr;
        e = moe::launch_tc_ffn(xg, offsets, counts, W_up, W_down, rows, d, d_ff, E, out, H, parts,
                               combine_reads_parts, status, kWaitTimeoutNs, sms, s, nullptr, act, b_up, b_down);
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core expert FFN launch");
        if (p.decode && combine_reads_parts) {
            if (parts_out) *parts_out = parts;
            if (nparts_out) *nparts_out = p.splits_down;
        }
        return MOE_OK;
    }
    e = moe::launch_simt_ffn(xg, offsets, counts, W_up, W_down, dt == MOE_BF16 ? 1 : 0, rows, d, d_ff,
                             E, out, H_keep ? H_keep : ffn_ws, s, act, b_up, b_down);
    if (e != cudaSuccess) return cuda_fail(e, "CUDA-core expert FFN launch");
    return MOE_OK;
}

// ---------------------------------------------------------------- dispatch without a workspace
// Scratch for moe_dispatch_noalloc: the per-block histograms and the
// per-(choice, expert) totals of the dispatch passes, in a fixed device array
// that every GPU loading this library holds until the process exits.
constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Unique id of the calling thread's current CUDA context (0 if there is none
// yet).  Context ids are never reused within a process, unlike the handles.
unsigned long long current_context_id() {
    static const auto fns = [] {
        struct F {
            PFN_cuCtxGetCurrent_v4000 get = nullptr;
            PFN_cuCtxGetId_v12000 id = nullptr;
        } f;
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f.get = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f.id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
        return f;
    }();
    if (fns.get == nullptr || fns.id == nullptr) return 0;
    CUcontext ctx = nullptr;
    if (fns.get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    unsigned long long id = 0;
    if (fns.id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_noalloc_scratch in the current device's context.  In
// host code the array's name is only a host-side stand-in, so the address is
// looked up with cudaGetSymbolAddress, with the device current, once per
// device and context: a new context (after cudaDeviceReset, say) reloads the
// module, which may place the array elsewhere, so its address is looked up
// again.
cudaError_t noalloc_scratch_address(void **out) {
    static std::mutex mu;
    static void *addr[64] = {nullptr};
    static unsigned long long ctx_of[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    const unsigned long long ctx = current_context_id();
    if (addr[dev] == nullptr || ctx == 0 || ctx != ctx_of[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // creates the context if needed
        if (e != cudaSuccess) return e;
        addr[dev] = p;
        ctx_of[dev] = current_context_id();
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

const char *moe_last_error(void) { return g_err.c_str(); }

int moe_num_sms(void) { return num_sms_current(); }

int64_t moe_capacity(int64_t N, int E, int k, double cf) {
    if (N < 0 || E < 1 || E > 256 || k < 1 || k > E || !(cf > 0.0)) return -1;
    if (std::isinf(cf)) return N;
    const double c = std::ceil(cf * static_cast<double>(N) * static_cast<double>(k) / static_cast<double>(E));
    if (c > static_cast<double>(N)) return N;
    return static_cast<int64_t>(c);
}

int64_t moe_gathered_rows(int64_t N, int E, int k, double cf) {
    const int64_t C = moe_capacity(N, E, k, cf);
    if (C < 0) return -1;
    return rows_for(N, E, k, C);
}

size_t moe_route_workspace_size(int d, int E) {
    if (d < 1 || E < 1 || E > 256) return 0;
    return moe::kStatusBytes + moe::route_tc_w3_bytes(d, E);
}

moe_status moe_route_ex(const void *x, moe_dtype dt, const float *W_g, const float *b_g,
                        const float *noise, float sigma, int64_t N, int d, int E, int k,
                        float *logits_out, int32_t *topk_idx, float *gates, void *ws, size_t ws_bytes,
                        void *stream) {
    moe_status st = check_shape(N, d, E, k, dt);
    if (st != MOE_OK) return st;
    if (N > 0) {
        REQUIRE_PTR(x, "x");
        REQUIRE_PTR(W_g, "W_g");
        REQUIRE_PTR(topk_idx, "topk_idx");
        REQUIRE_PTR(gates, "gates");
        OPTIONAL_PTR(b_g, "b_g");
        OPTIONAL_PTR(noise, "noise");
        OPTIONAL_PTR(logits_out, "logits_out");
    }
    OPTIONAL_PTR(ws, "ws");
    if (ws != nullptr && ws_bytes < static_cast<size_t>(moe::kStatusBytes))
        return fail(MOE_ERR_WORKSPACE, "router workspace needs at least %d bytes (got %zu)", moe::kStatusBytes,
                    ws_bytes);
    if (!std::isfinite(sigma)) return fail(MOE_ERR_INVALID_ARG, "sigma must be finite");
    // a workspace large enough for the split router weights: the pre-split path of moe_forward
    const size_t w3 = moe::route_tc_w3_bytes(d, E);
    void *w3p = (ws != nullptr && dt == MOE_BF16 && w3 > 0 && ws_bytes >= moe::kStatusBytes + w3)
                    ? static_cast<void *>(static_cast<uint8_t *>(ws) + moe::kStatusBytes)
                    : nullptr;
    cudaError_t e = moe::launch_route(x, dt == MOE_BF16 ? 1 : 0, W_g, b_g, noise, sigma, N, d, E, k,
                                      logits_out, topk_idx, gates, static_cast<uint32_t *>(ws),
                                      static_cast<cudaStream_t>(stream), w3p);
    if (e != cudaSuccess) return cuda_fail(e, "router launch");
    return MOE_OK;
}

moe_status moe_route(const void *x, moe_dtype dt, const float *W_g, const float *b_g,
                     const float *noise, float sigma, int64_t N, int d, int E, int k,
                     float *logits_out, int32_t *topk_idx, float *gates, void *stream) {
    return moe_route_ex(x, dt, W_g, b_g, noise, sigma, N, d, E, k, logits_out, topk_idx, gates, nullptr, 0, stream);
}

moe_status moe_check_route_status(void *stream, uint32_t *detail) {
    uint32_t word = 0;
    cudaError_t e = moe::route_status_read_clear(&word, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "router status read");
    if (detail) *detail = word;
    if (word & moe::ST_TIMEOUT)
        return fail(MOE_ERR_TIMEOUT, "a router wait ran out (status 0x%08x)", word);
    if (word & moe::ST_BOUNDS)
        return fail(MOE_ERR_DEVICE_CHECK, "a router index check failed (status 0x%08x)", word);
    return MOE_OK;
}

size_t moe_dispatch_workspace_size(int64_t N, int E, int k) {
    if (N < 0 || E < 1 || k < 1) return 0;
    return moe::dispatch_ws_bytes(N, E, k);
}

moe_status moe_dispatch(const int32_t *topk_idx, const void *x, moe_dtype dt, int64_t N, int d,
                        int E, int k, double cf, int32_t *slot, int32_t *counts,
                        int32_t *offsets, void *x_gathered, void *ws, size_t ws_bytes,
                        void *stream) {
    moe_status st = check_shape(N, d, E, k, dt);
    if (st != MOE_OK) return st;
    const int64_t C = moe_capacity(N, E, k, cf);
    if (C < 0) return fail(MOE_ERR_INVALID_ARG, "capacity factor must be > 0 or +inf (got %g)", cf);
    REQUIRE_PTR(counts, "counts");
    REQUIRE_PTR(offsets, "offsets");
    if (N > 0) {
        REQUIRE_PTR(topk_idx, "topk_idx");
        REQUIRE_PTR(x, "x");
        REQUIRE_PTR(slot, "slot");
        REQUIRE_PTR(x_gathered, "x_gathered");
    }
    const size_t need = moe::dispatch_ws_bytes(N, E, k);
    if (ws == nullptr || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "dispatch workspace needs %zu bytes (got %zu)", need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    REQUIRE_PTR(ws, "ws");
    cudaError_t e = moe::launch_dispatch(topk_idx, x, elem_bytes(dt), N, d, E, k, C, slot, counts,
                                         offsets, x_gathered, ws, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    return MOE_OK;
}

moe_status moe_dispatch_noalloc(const int32_t *topk_idx, const void *x, moe_dtype dt, int64_t N, int d,
                                int E, int k, double cf, int32_t *slot, int32_t *counts,
                                int32_t *offsets, void *x_gathered, void *stream) {
    moe_status st = check_shape(N, d, E, k, dt);
    if (st != MOE_OK) return st;
    const int64_t C = moe_capacity(N, E, k, cf);
    if (C < 0) return fail(MOE_ERR_INVALID_ARG, "capacity factor must be > 0 or +inf (got %g)", cf);
    REQUIRE_PTR(counts, "counts");
    REQUIRE_PTR(offsets, "offsets");
    if (N > 0) {
        REQUIRE_PTR(topk_idx, "topk_idx");
        REQUIRE_PTR(x, "x");
        REQUIRE_PTR(slot, "slot");
        REQUIRE_PTR(x_gathered, "x_gathered");
    }
    const size_t need = moe::dispatch_ws_bytes(N, E, k);
    if (need > kNoAllocScratchBytes)
        return fail(MOE_ERR_INVALID_ARG,
                    "moe_dispatch_noalloc: N=%lld, E=%d, k=%d needs %zu bytes of scratch, more than its "
                    "fixed %zu bytes; use moe_dispatch with a workspace",
                    (long long)N, E, k, need, kNoAllocScratchBytes);
    void *scratch = nullptr;
    cudaError_t e = noalloc_scratch_address(&scratch);
    if (e != cudaSuccess) return cuda_fail(e, "moe_dispatch_noalloc scratch lookup");
    e = moe::launch_dispatch(topk_idx, x, elem_bytes(dt), N, d, E, k, C, slot, counts, offsets, x_gathered,
                             scratch, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    return MOE_OK;
}

size_t moe_shard_workspace_size(int64_t N_local, int E, int k) {
    if (N_local < 0 || E < 1 || k < 1) return 0;
    return moe::dispatch_ws_bytes(N_local, E, k);
}

moe_status moe_shard_count(const int32_t *topk_idx, int64_t N_local, int E, int k, int32_t *counts_je,
                           void *ws, size_t ws_bytes, void *stream) {
    moe_status st = check_shape(N_local, 1, E, k, MOE_BF16);
    if (st != MOE_OK) return st;
    REQUIRE_PTR(counts_je, "counts_je");
    if (N_local > 0) REQUIRE_PTR(topk_idx, "topk_idx");
    const size_t need = moe::dispatch_ws_bytes(N_local, E, k);
    if (ws == nullptr || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "shard workspace needs %zu bytes (got %zu)", need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    REQUIRE_PTR(ws, "ws");
    cudaError_t e = moe::launch_shard_count(topk_idx, N_local, E, k, counts_je, ws, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "shard count launch");
    return MOE_OK;
}

moe_status moe_shard_base(const int32_t *all_counts, int G, int rank, int E, int k, int32_t *base,
                          void *stream) {
    if (G < 1 || rank < 0 || rank >= G) return fail(MOE_ERR_INVALID_ARG, "need 0 <= rank < G (got rank=%d, G=%d)", rank, G);
    if (E < 1 || E > 256 || k < 1 || k > E) return fail(MOE_ERR_INVALID_ARG, "bad E or k");
    REQUIRE_PTR(all_counts, "all_counts");
    REQUIRE_PTR(base, "base");
    cudaError_t e = moe::launch_shard_base(all_counts, G, rank, E, k, base, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "shard base launch");
    return MOE_OK;
}

moe_status moe_shard_dispatch(const int32_t *topk_idx, const void *x, moe_dtype dt, int64_t N_local, int d,
                              int E, int k, int64_t C, const int32_t *counts_je, const int32_t *base,
                              int32_t *slot, int32_t *counts, int32_t *offsets, void *x_gathered, void *ws,
                              size_t ws_bytes, void *stream) {
    moe_status st = check_shape(N_local, d, E, k, dt);
    if (st != MOE_OK) return st;
    if (C < 0) return fail(MOE_ERR_INVALID_ARG, "capacity must be >= 0 (got %lld)", (long long)C);
    REQUIRE_PTR(counts, "counts");
    REQUIRE_PTR(offsets, "offsets");
    if (N_local > 0) {
        REQUIRE_PTR(topk_idx, "topk_idx");
        REQUIRE_PTR(x, "x");
        REQUIRE_PTR(counts_je, "counts_je");
        REQUIRE_PTR(base, "base");
        REQUIRE_PTR(slot, "slot");
        REQUIRE_PTR(x_gathered, "x_gathered");
    }
    const size_t need = moe::dispatch_ws_bytes(N_local, E, k);
    if (ws == nullptr || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "shard workspace needs %zu bytes (got %zu)", need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    REQUIRE_PTR(ws, "ws");
    cudaError_t e = moe::launch_shard_dispatch(topk_idx, x, elem_bytes(dt), N_local, d, E, k, C, counts_je, base,
                                               slot, counts, offsets, x_gathered, ws,
                                               static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "shard dispatch launch");
    return MOE_OK;
}

size_t moe_expert_ffn_workspace_size(int64_t rows, int d, int E, int d_ff, moe_dtype dt) {
    if (rows < 0 || d < 1 || E < 1 || d_ff < 1 || (dt != MOE_F32 && dt != MOE_BF16)) return 0;
    return moe::kStatusBytes + ffn_ws_bytes(rows, d, E, d_ff, dt);
}

moe_status moe_expert_ffn_ex(const void *x_gathered, const int32_t *offsets, const int32_t *counts,
                             const void *W_up, const void *W_down, moe_dtype dt, int64_t rows, int d,
                             int d_ff, int E, int activation, const float *b_up, const float *b_down,
                             void *out_gathered, void *ws, size_t ws_bytes, void *stream) {
    if (dt != MOE_F32 && dt != MOE_BF16) return fail(MOE_ERR_INVALID_ARG, "dtype must be MOE_F32 or MOE_BF16");
    if (activation != MOE_ACT_RELU && activation != MOE_ACT_GELU)
        return fail(MOE_ERR_INVALID_ARG, "activation must be MOE_ACT_RELU or MOE_ACT_GELU");
    if (rows < 0 || rows % 128 != 0)
        return fail(MOE_ERR_INVALID_ARG, "rows must be a non-negative multiple of 128 (moe_gathered_rows)");
    if (d < 1 || d_ff < 1 || E < 1 || E > 256) return fail(MOE_ERR_INVALID_ARG, "bad d, d_ff or E");
    if (rows > INT32_MAX) return fail(MOE_ERR_INVALID_ARG, "rows must fit in int32");
    REQUIRE_PTR(offsets, "offsets");
    REQUIRE_PTR(counts, "counts");
    REQUIRE_PTR(W_up, "W_up");
    REQUIRE_PTR(W_down, "W_down");
    OPTIONAL_PTR(b_up, "b_up");
    OPTIONAL_PTR(b_down, "b_down");
    if (rows > 0) {
        REQUIRE_PTR(x_gathered, "x_gathered");
        REQUIRE_PTR(out_gathered, "out_gathered");
    }
    const size_t need = moe::kStatusBytes + ffn_ws_bytes(rows, d, E, d_ff, dt);
    if (ws == nullptr || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "expert FFN workspace needs %zu bytes (got %zu)", need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    REQUIRE_PTR(ws, "ws");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t *status = static_cast<uint32_t *>(ws);
    if (rows == 0) return MOE_OK;
    return run_ffn(x_gathered, offsets, counts, W_up, W_down, dt, rows, d, d_ff, E, out_gathered,
                   static_cast<uint8_t *>(ws) + moe::kStatusBytes, false, nullptr, nullptr, status, s, activation,
                   b_up, b_down);
}

moe_status moe_expert_ffn_train(const void *x_gathered, const int32_t *offsets, const int32_t *counts,
                                const void *W_up, const void *W_down, moe_dtype dt, int64_t rows, int d,
                                int d_ff, int E, void *out_gathered, void *H, void *ws, size_t ws_bytes,
                                void *stream) {
    if (dt != MOE_F32 && dt != MOE_BF16) return fail(MOE_ERR_INVALID_ARG, "dtype must be MOE_F32 or MOE_BF16");
    if (rows < 0 || rows % 128 != 0)
        return fail(MOE_ERR_INVALID_ARG, "rows must be a non-negative multiple of 128 (moe_gathered_rows)");
    if (d < 1 || d_ff < 1 || E < 1 || E > 256) return fail(MOE_ERR_INVALID_ARG, "bad d, d_ff or E");
    if (rows > INT32_MAX) return fail(MOE_ERR_INVALID_ARG, "rows must fit in int32");
    REQUIRE_PTR(offsets, "offsets");
    REQUIRE_PTR(counts, "counts");
    REQUIRE_PTR(W_up, "W_up");
    REQUIRE_PTR(W_down, "W_down");
    if (rows > 0) {
        REQUIRE_PTR(x_gathered, "x_gathered");
        REQUIRE_PTR(out_gathered, "out_gathered");
        REQUIRE_PTR(H, "H");
    }
    const size_t need = moe::kStatusBytes + ffn_ws_bytes(rows, d, E, d_ff, dt);
    if (ws == nullptr || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "expert FFN workspace needs %zu bytes (got %zu)", need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    REQUIRE_PTR(ws, "ws");
    if (rows == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return run_ffn(x_gathered, offsets, counts, W_up, W_down, dt, rows, d, d_ff, E, out_gathered,
                   static_cast<uint8_t *>(ws) + moe::kStatusBytes, false, nullptr, nullptr,
                   static_cast<uint32_t *>(ws), s, MOE_ACT_RELU, nullptr, nullptr, H);
}

size_t moe_backward_workspace_size(int64_t N, int d, int E, int d_ff, int k, int64_t rows, moe_dtype dt) {
    if (check_shape(N, d, E, k, dt) != MOE_OK || d_ff < 1 || rows < 0) return 0;
    moe::BwdArgs a{};
    a.dt = dt == MOE_BF16 ? 1 : 0;
    a.N = N; a.d = d; a.E = E; a.d_ff = d_ff; a.k = k; a.rows = rows;
    return moe::bwd_layout(a, num_sms_current()).total;
}

moe_status moe_backward(const void *x, moe_dtype dt, const float *W_g, const void *W_up, const void *W_down,
                        int64_t N, int d, int E, int d_ff, int k, int64_t rows, const int32_t *topk_idx,
                        const float *gates, const int32_t *slot, const int32_t *offsets, const int32_t *counts,
                        const void *x_gathered, const void *H, const void *out_gathered, const void *dy,
                        void *dx, float *dW_g, float *db_g, float *dW_up, float *dW_down, void *ws,
                        size_t ws_bytes, void *stream) {
    moe_status st = check_shape(N, d, E, k, dt);
    if (st != MOE_OK) return st;
    if (d_ff < 1) return fail(MOE_ERR_INVALID_ARG, "d_ff must be >= 1");
    if (rows < 0 || rows % 128 != 0 || rows > INT32_MAX)
        return fail(MOE_ERR_INVALID_ARG, "rows must be a non-negative multiple of 128 that fits in int32");
    REQUIRE_PTR(W_g, "W_g");
    REQUIRE_PTR(W_up, "W_up");
    REQUIRE_PTR(W_down, "W_down");
    REQUIRE_PTR(dW_g, "dW_g");
    REQUIRE_PTR(db_g, "db_g");
    REQUIRE_PTR(dW_up, "dW_up");
    REQUIRE_PTR(dW_down, "dW_down");
    REQUIRE_PTR(offsets, "offsets");
    REQUIRE_PTR(counts, "counts");
    if (N > 0) {
        REQUIRE_PTR(x, "x");
        REQUIRE_PTR(topk_idx, "topk_idx");
        REQUIRE_PTR(gates, "gates");
        REQUIRE_PTR(slot, "slot");
        REQUIRE_PTR(dy, "dy");
        REQUIRE_PTR(dx, "dx");
        REQUIRE_PTR(x_gathered, "x_gathered");
        REQUIRE_PTR(H, "H");
        REQUIRE_PTR(out_gathered, "out_gathered");
    }
    moe::BwdArgs a{x, dt == MOE_BF16 ? 1 : 0, W_g, W_up, W_down, N, d, E, d_ff, k, rows, topk_idx, gates, slot,
                   offsets, counts, x_gathered, H, out_gathered, dy, dx, dW_g, db_g, dW_up, dW_down};
    const int sms = num_sms_current();
    const size_t need = moe::bwd_layout(a, sms).total;
    if (ws == nullptr || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "backward workspace needs %zu bytes (got %zu)", need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    REQUIRE_PTR(ws, "ws");
    cudaError_t e = moe::launch_backward(a, ws, static_cast<uint32_t *>(ws), kWaitTimeoutNs, sms,
                                         use_tensor_cores(dt, d, d_ff), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return MOE_OK;
}

moe_status moe_expert_ffn(const void *x_gathered, const int32_t *offsets, const int32_t *counts,
                          const void *W_up, const void *W_down, moe_dtype dt, int64_t rows,
                          int d, int d_ff, int E, void *out_gathered, void *ws, size_t ws_bytes,
                          void *stream) {
    return moe_expert_ffn_ex(x_gathered, offsets, counts, W_up, W_down, dt, rows, d, d_ff, E, MOE_ACT_RELU,
                             nullptr, nullptr, out_gathered, ws, ws_bytes, stream);
}

moe_status moe_combine(const void *out_gathered, const int32_t *slot, const int32_t *topk_idx,
                       const int32_t *offsets, const float *gates, moe_dtype dt, int64_t N,
                       int d, int k, void *y, void *stream) {
    if (dt != MOE_F32 && dt != MOE_BF16) return fail(MOE_ERR_INVALID_ARG, "dtype must be MOE_F32 or MOE_BF16");
    if (N < 0 || d < 1 || k < 1 || k > 256) return fail(MOE_ERR_INVALID_ARG, "bad N, d or k");
    if (N > 0) {
        REQUIRE_PTR(slot, "slot");
        REQUIRE_PTR(topk_idx, "topk_idx");
        REQUIRE_PTR(offsets, "offsets");
        REQUIRE_PTR(gates, "gates");
        REQUIRE_PTR(y, "y");
        OPTIONAL_PTR(out_gathered, "out_gathered");
    }
    cudaError_t e = moe::launch_combine(out_gathered, nullptr, 0, 0, slot, topk_idx, offsets, gates,
                                        dt == MOE_BF16 ? 1 : 0, N, d, k, 256, y,
                                        static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    return MOE_OK;
}

size_t moe_load_stats_workspace_size(void) { return moe::stats_ws_bytes(); }

moe_status moe_load_stats(const int32_t *topk_idx, const float *gates, int64_t N, int E, int k, double cf,
                          int32_t *load, int32_t *used, double *importance, void *ws, size_t ws_bytes,
                          void *stream) {
    if (N < 0 || E < 1 || E > moe::kStatsMaxE || k < 1 || k > E)
        return fail(MOE_ERR_INVALID_ARG, "need N >= 0 and 1 <= k <= E <= %d", moe::kStatsMaxE);
    if (N * static_cast<int64_t>(k) >= (static_cast<int64_t>(1) << 31))
        return fail(MOE_ERR_INVALID_ARG, "N * k must be below 2^31");
    const int64_t C = moe_capacity(N, E, k, cf);
    if (C < 0) return fail(MOE_ERR_INVALID_ARG, "capacity factor must be > 0 or +inf (got %g)", cf);
    if (N > 0) REQUIRE_PTR(topk_idx, "topk_idx");
    OPTIONAL_PTR(gates, "gates");
    REQUIRE_PTR(load, "load");
    REQUIRE_PTR(used, "used");
    OPTIONAL_PTR(importance, "importance");
    if (ws == nullptr || ws_bytes < moe::stats_ws_bytes())
        return fail(MOE_ERR_WORKSPACE, "load statistics need %zu bytes of workspace", moe::stats_ws_bytes());
    REQUIRE_PTR(ws, "ws");
    cudaError_t e = moe::launch_load_stats(topk_idx, gates, N, E, k, C, load, used, importance, ws,
                                           static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "load statistics launch");
    return MOE_OK;
}

size_t moe_workspace_size(int64_t N, int d, int E, int d_ff, int k, double cf, moe_dtype dt) {
    if (check_shape(N, d, E, k, dt) != MOE_OK || d_ff < 1) return 0;
    const int64_t C = moe_capacity(N, E, k, cf);
    if (C < 0) return 0;
    return forward_layout(N, d, E, d_ff, k, rows_for(N, E, k, C), dt).total;
}

moe_status moe_forward_ex(const void *x, moe_dtype dt, const float *W_g, const float *b_g,
                          const float *noise, float sigma, int64_t N, int d, int E, int d_ff,
                          int k, double cf, const void *W_up, const void *W_down, int activation,
                          const float *b_up, const float *b_down, void *y,
                          float *logits_out, int32_t *topk_out, float *gates_out,
                          int32_t *slot_out, int32_t *counts_out,
                          void *ws, size_t ws_bytes, void *stream) {
    moe_status st = check_shape(N, d, E, k, dt);
    if (st != MOE_OK) return st;
    if (d_ff < 1) return fail(MOE_ERR_INVALID_ARG, "d_ff must be >= 1");
    const int64_t C = moe_capacity(N, E, k, cf);
    if (C < 0) return fail(MOE_ERR_INVALID_ARG, "capacity factor must be > 0 or +inf (got %g)", cf);
    if (!std::isfinite(sigma)) return fail(MOE_ERR_INVALID_ARG, "sigma must be finite");
    if (activation != MOE_ACT_RELU && activation != MOE_ACT_GELU)
        return fail(MOE_ERR_INVALID_ARG, "activation must be MOE_ACT_RELU or MOE_ACT_GELU");
    OPTIONAL_PTR(b_up, "b_up");
    OPTIONAL_PTR(b_down, "b_down");
    REQUIRE_PTR(W_g, "W_g");
    REQUIRE_PTR(W_up, "W_up");
    REQUIRE_PTR(W_down, "W_down");
    if (N > 0) {
        REQUIRE_PTR(x, "x");
        REQUIRE_PTR(y, "y");
    }
    OPTIONAL_PTR(b_g, "b_g");
    OPTIONAL_PTR(noise, "noise");
    OPTIONAL_PTR(logits_out, "logits_out");
    OPTIONAL_PTR(topk_out, "topk_out");
    OPTIONAL_PTR(gates_out, "gates_out");
    OPTIONAL_PTR(slot_out, "slot_out");
    OPTIONAL_PTR(counts_out, "counts_out");
    const int64_t rows = rows_for(N, E, k, C);
    if (rows > INT32_MAX) return fail(MOE_ERR_INVALID_ARG, "gathered rows must fit in int32");
    const FwdLayout L = forward_layout(N, d, E, d_ff, k, rows, dt);
    if (ws == nullptr || ws_bytes < L.total)
        return fail(MOE_ERR_WORKSPACE, "forward workspace needs %zu bytes (got %zu)", L.total,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    REQUIRE_PTR(ws, "ws");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *w = static_cast<uint8_t *>(ws);
    uint32_t *status = reinterpret_cast<uint32_t *>(w + L.status);
    int32_t *topk = topk_out ? topk_out : reinterpret_cast<int32_t *>(w + L.topk);
    float *gates = gates_out ? gates_out : reinterpret_cast<float *>(w + L.gates);
    int32_t *slot = slot_out ? slot_out : reinterpret_cast<int32_t *>(w + L.slot);
    int32_t *counts = counts_out ? counts_out : reinterpret_cast<int32_t *>(w + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(w + L.offsets);
    void *xg = w + L.xg;
    void *og = w + L.og;

    if (N > 0 && L.total > L.fused &&
        use_fused_decode(x, W_g, N, d, E, d_ff, k, rows, dt, activation, b_up, b_down)) {
        const int sms = num_sms_current();
        const moe::TcPlan p = moe::plan_tc_ffn(rows, d, d_ff, E, sms);
        uint8_t *f = w + L.ffn;
        float *parts_dn = reinterpret_cast<float *>(f + moe::align_up(static_cast<size_t>(rows) * d_ff * 2, 256));
        float *parts_up = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(parts_dn) +
                                                    moe::align_up(static_cast<size_t>(p.splits_down) * rows * d * 4, 256));
        cudaError_t e = moe::launch_decode_fused(x, W_g, b_g, noise, sigma, N, d, E, d_ff, k, C, W_up, W_down, y,
                                                 logits_out, topk, gates, slot, counts, offsets, xg, rows, f, parts_dn,
                                                 parts_up, p.splits_up, p.splits_down, w + L.fused, status,
                                                 kWaitTimeoutNs, sms, s);
        if (e != cudaSuccess) return cuda_fail(e, "fused small-batch layer launch");
        return MOE_OK;
    }
    void *w3 = (L.xg > L.w3) ? static_cast<void *>(w + L.w3) : nullptr;
    cudaError_t e = moe::launch_route(x, dt == MOE_BF16 ? 1 : 0, W_g, b_g, noise, sigma, N, d, E, k,
                                      logits_out, topk, gates, status, s, w3);
    if (e != cudaSuccess) return cuda_fail(e, "router launch");
    if (N == 0) {
        if (counts_out) {
            e = cudaMemsetAsync(counts_out, 0, sizeof(int32_t) * E, s);
            if (e != cudaSuccess) return cuda_fail(e, "counts reset");
        }
        return MOE_OK;
    }
    e = moe::launch_dispatch(topk, x, elem_bytes(dt), N, d, E, k, C, slot, counts, offsets, xg,
                             w + L.dws, s);
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    float *parts = nullptr;
    int nparts = 0;
    st = run_ffn(xg, offsets, counts, W_up, W_down, dt, rows, d, d_ff, E, og, w + L.ffn, true, &parts,
                 &nparts, status, s, activation, b_up, b_down);
    if (st != MOE_OK) return st;
    e = moe::launch_combine(og, parts, nparts, rows * static_cast<int64_t>(d), slot, topk, offsets,
                            gates, dt == MOE_BF16 ? 1 : 0, N, d, k, E, y, s, nparts > 0 ? b_down : nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    return MOE_OK;
}

moe_status moe_forward(const void *x, moe_dtype dt, const float *W_g, const float *b_g,
                       const float *noise, float sigma, int64_t N, int d, int E, int d_ff,
                       int k, double cf, const void *W_up, const void *W_down, void *y,
                       float *logits_out, int32_t *topk_out, float *gates_out,
                       int32_t *slot_out, int32_t *counts_out,
                       void *ws, size_t ws_bytes, void *stream) {
    return moe_forward_ex(x, dt, W_g, b_g, noise, sigma, N, d, E, d_ff, k, cf, W_up, W_down, MOE_ACT_RELU,
                          nullptr, nullptr, y, logits_out, topk_out, gates_out, slot_out, counts_out, ws,
                          ws_bytes, stream);
}

int moe_forward_launches(int64_t N, int d, int E, int d_ff, int k, double cf, moe_dtype dt) {
    if (check_shape(N, d, E, k, dt) != MOE_OK || d_ff < 1 || moe_capacity(N, E, k, cf) < 0) return -1;
    if (N == 0) return 0;
    if (use_fused_decode(nullptr, nullptr, N, d, E, d_ff, k, rows_for(N, E, k, moe_capacity(N, E, k, cf)), dt,
                         MOE_ACT_RELU, nullptr, nullptr))
        return 1;
    int ffn = 2;
    if (use_tensor_cores(dt, d, d_ff)) {
        const int64_t rows = rows_for(N, E, k, moe_capacity(N, E, k, cf));
        ffn = moe::tc_ffn_launches(moe::plan_tc_ffn(rows, d, d_ff, E, num_sms_current()), true);
    }
    // router (+ its weight split) + dispatch passes + expert FFN + combine
    const bool w3 = dt == MOE_BF16 && moe::route_tc_w3_bytes(d, E) > 0;
    return moe::route_launches(dt == MOE_BF16 ? 1 : 0, N, d, E, k, w3) + moe::dispatch_launches(N, E, k) + ffn + 1;
}

int moe_set_fused_small_batch(int on) {
    const int prev = fused_decode_enabled() ? 1 : 0;
    if (on >= 0) g_fused_small_batch.store(on != 0 ? 1 : 0, std::memory_order_relaxed);
    return prev;
}

moe_status moe_check_status(void *ws, void *stream, uint32_t *detail) {
    if (ws == nullptr) return fail(MOE_ERR_INVALID_ARG, "ws must not be NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    e = cudaMemsetAsync(ws, 0, sizeof word, s);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    if (detail) *detail = word;
    if (word & moe::ST_TIMEOUT)
        return fail(MOE_ERR_TIMEOUT, "a kernel's bounded wait ran out (status 0x%08x)", word);
    if (word & moe::ST_BOUNDS)
        return fail(MOE_ERR_DEVICE_CHECK, "a kernel's index check failed (status 0x%08x)", word);
    return MOE_OK;
}

moe_status moe_debug_wait_timeout(uint32_t timeout_us, void *ws, size_t ws_bytes, void *stream) {
    if (ws == nullptr || ws_bytes < static_cast<size_t>(moe::kStatusBytes))
        return fail(MOE_ERR_WORKSPACE, "needs a workspace of at least %d bytes", moe::kStatusBytes);
    if (timeout_us == 0 || timeout_us > 2000000u)
        return fail(MOE_ERR_INVALID_ARG, "timeout_us must be in [1, 2000000]");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e =
        moe::launch_wait_timeout(static_cast<uint32_t *>(ws), static_cast<uint64_t>(timeout_us) * 1000ull, s);
    if (e != cudaSuccess) return cuda_fail(e, "wait-timeout diagnostic launch");
    return MOE_OK;
}

}  // extern "C"
