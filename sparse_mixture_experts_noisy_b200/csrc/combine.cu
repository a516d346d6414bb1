// Gate-weighted combine back to token order.
//
// "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 11 (g_i E_i(x)) and
// STEP 12 (y = sum_i g_i E_i(x)); "nanoMoEの深層解剖" slides 38-40 (output =
// cb_weight @ exp_out: a dropped pair has weight 0, the kept ones keep their
// gate, so a token whose choices were all dropped gets a zero row).
// The dense [tokens, E*C] x [E*C, d] product of the slides is replaced by a
// gather: for each token, threads own chunks of its output columns, read those
// chunks of the token's k expert-output rows and accumulate g * row in fp32, in
// choice order j = 0..k-1.  Small batches give a token to a whole block in
// turn; large ones give each thread one chunk of one token.
//
// The expert outputs are either rows of dtype T (one partial) or `parts`
// fp32 partial sums over K-splits of the down projection, which are added in
// split order before the gate is applied.
#include "common.cuh"
#include "internal.h"

#include <cstdlib>

namespace moe {

namespace {

template <typename T, int VEC>
struct Vec;
template <>
struct Vec<__nv_bfloat16, 8> {
    using Raw = uint4;
    static __device__ __forceinline__ Raw load_raw(const __nv_bfloat16 *p) { return *reinterpret_cast<const uint4 *>(p); }
    static __device__ __forceinline__ void widen(const Raw &u, float (&v)[8]) {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[8]) {
        uint4 u = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&v)[8]) {
        uint4 u;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        *reinterpret_cast<uint4 *>(p) = u;
    }
};
template <>
struct Vec<float, 4> {
    using Raw = float4;
    static __device__ __forceinline__ Raw load_raw(const float *p) { return *reinterpret_cast<const float4 *>(p); }
    static __device__ __forceinline__ void widen(const Raw &u, float (&v)[4]) {
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
    static __device__ __forceinline__ void load(const float *p, float (&v)[4]) {
        float4 u = *reinterpret_cast<const float4 *>(p);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
    static __device__ __forceinline__ void store(float *p, const float (&v)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <typename T>
struct Vec<T, 1> {
    using Raw = T;
    static __device__ __forceinline__ Raw load_raw(const T *p) { return *p; }
    static __device__ __forceinline__ void widen(const Raw &u, float (&v)[1]) { v[0] = to_f32<T>(u); }
    static __device__ __forceinline__ void load(const T *p, float (&v)[1]) { v[0] = to_f32<T>(*p); }
    static __device__ __forceinline__ void store(T *p, const float (&v)[1]) { *p = from_f32<T>(v[0]); }
};

template <int VEC>
__device__ __forceinline__ void load_f32(const float *p, float (&v)[VEC]) {
    if constexpr (VEC == 8) {
        float4 a = *reinterpret_cast<const float4 *>(p);
        float4 b = *reinterpret_cast<const float4 *>(p + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else if constexpr (VEC == 4) {
        float4 a = *reinterpret_cast<const float4 *>(p);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else {
        v[0] = *p;
    }
}

template <typename T, int VEC>
__global__ void __launch_bounds__(256)
combine_kernel(const T *__restrict__ out_rows, const float *__restrict__ parts, int nparts,
               int64_t part_stride, const int32_t *__restrict__ slot,
               const int32_t *__restrict__ topk_idx, const int32_t *__restrict__ offsets,
               const float *__restrict__ gates, int64_t N, int d, int k, int E,
               T *__restrict__ y, const float *__restrict__ b_down) {
    pdl_trigger();
    pdl_wait();
    // a block takes tokens in turn; its threads split the token's columns into
    // VEC-wide chunks; the token's k (row, gate) pairs are read once per block
    extern __shared__ int32_t c_smem[];
    int32_t *rows = c_smem;                                  // [k] source row or -1
    float *g = reinterpret_cast<float *>(rows + k);          // [k]
    int32_t *re = rows + 2 * k;                              // [k] expert
    const int chunks = d / VEC;
    for (int64_t t = blockIdx.x; t < N; t += gridDim.x) {
        for (int j = threadIdx.x; j < k; j += blockDim.x) {
            const int32_t sl = slot[t * k + j];
            const int32_t e = topk_idx[t * k + j];
            const bool ok = sl >= 0 && e >= 0 && e < E;
            rows[j] = ok ? offsets[e] + sl : -1;
            g[j] = ok ? gates[t * k + j] : 0.0f;
            re[j] = ok ? e : 0;
        }
        __syncthreads();
        for (int ch = threadIdx.x; ch < chunks; ch += blockDim.x) {
            const int c = ch * VEC;
            float acc[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[v] = 0.0f;
            for (int j = 0; j < k; ++j) {
                const int32_t r = rows[j];
                if (r < 0) continue;
                float o[VEC];
                if (nparts == 0) {
                    Vec<T, VEC>::load(out_rows + static_cast<int64_t>(r) * d + c, o);
                } else {
                    load_f32<VEC>(parts + static_cast<int64_t>(r) * d + c, o);
#pragma unroll 4
                    for (int p = 1; p < nparts; ++p) {
                        float q[VEC];
                        load_f32<VEC>(parts + p * part_stride + static_cast<int64_t>(r) * d + c, q);
#pragma unroll
                        for (int v = 0; v < VEC; ++v) o[v] += q[v];
                    }
                    if (b_down != nullptr) {
                        float bq[VEC];
                        load_f32<VEC>(b_down + static_cast<int64_t>(re[j]) * d + c, bq);
#pragma unroll
                        for (int v = 0; v < VEC; ++v) o[v] += bq[v];
                    }
                }
                const float gj = g[j];
#pragma unroll
                for (int v = 0; v < VEC; ++v) acc[v] = fmaf(gj, o[v], acc[v]);
            }
            Vec<T, VEC>::store(y + t * d + c, acc);
        }
        __syncthreads();
    }
}

// Large batches: each thread owns one VEC-wide chunk of one token's output
// (blocks of 128 chunks; a token spans ceil(d / VEC / 128) blocks).  The
// thread fetches the (slot, expert, gate) of up to kCombineGroup choices at
// once, then their row offsets, then their data, so a token costs three
// dependent memory round trips per group of choices rather than three per
// choice; the adds still run in choice order j = 0..k-1, the same arithmetic
// per element as the block kernel above.  Rows are dtype (nparts == 0).
constexpr int kCombineGroup = 6;

template <typename T, int VEC>
__global__ void __launch_bounds__(128, 6)
combine_token_kernel(const T *__restrict__ out_rows, const int32_t *__restrict__ slot,
                     const int32_t *__restrict__ topk_idx, const int32_t *__restrict__ offsets,
                     const float *__restrict__ gates, int64_t N, int d, int k, int E, int blocks_per_token,
                     T *__restrict__ y) {
    pdl_trigger();
    pdl_wait();
    const int64_t t = blockIdx.x / blocks_per_token;
    const int c = ((blockIdx.x % blocks_per_token) * 128 + threadIdx.x) * VEC;
    if (t >= N || c >= d) return;
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.0f;
    for (int j0 = 0; j0 < k; j0 += kCombineGroup) {
        int32_t sl[kCombineGroup], ex[kCombineGroup];
        float g[kCombineGroup];
#pragma unroll
        for (int i = 0; i < kCombineGroup; ++i) {
            const int j = j0 + i;
            sl[i] = -1;
            if (j < k) {
                sl[i] = slot[t * k + j];
                ex[i] = topk_idx[t * k + j];
                g[i] = gates[t * k + j];
            }
        }
        int32_t r[kCombineGroup];
#pragma unroll
        for (int i = 0; i < kCombineGroup; ++i) {
            const bool ok = sl[i] >= 0 && ex[i] >= 0 && ex[i] < E;
            r[i] = ok ? offsets[ex[i]] + sl[i] : -1;
        }
        typename Vec<T, VEC>::Raw raw[kCombineGroup];
#pragma unroll
        for (int i = 0; i < kCombineGroup; ++i)
            if (r[i] >= 0) raw[i] = Vec<T, VEC>::load_raw(out_rows + static_cast<int64_t>(r[i]) * d + c);
#pragma unroll
        for (int i = 0; i < kCombineGroup; ++i)
            if (r[i] >= 0) {
                float o[VEC];
                Vec<T, VEC>::widen(raw[i], o);
#pragma unroll
                for (int v = 0; v < VEC; ++v) acc[v] = fmaf(g[i], o[v], acc[v]);
            }
    }
    Vec<T, VEC>::store(y + t * d + c, acc);
}

// Large batches: one warp per token (grid-stride), the mirror of the gather.
// Lanes j < k fetch the token's (row, gate) pairs once and pass them round by
// shuffles.  Each pass loads U 16-byte chunks per lane of every kept row
// before using any (k * U loads in flight per lane, kept packed), then forms
// the weighted sums in choice order (the same arithmetic per element as the
// kernels above) and stores U chunks of y.
template <typename T, int VEC, int KMAX, int U>
__global__ void __launch_bounds__(256, 3)
combine_warp_kernel(const T *__restrict__ out_rows, const int32_t *__restrict__ slot,
                    const int32_t *__restrict__ topk_idx, const int32_t *__restrict__ offsets,
                    const float *__restrict__ gates, int64_t N, int d, int k, int E, T *__restrict__ y) {
    using Raw = typename Vec<T, VEC>::Raw;
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int chunks = d / VEC;
    for (int64_t t = w0; t < N; t += nw) {
        int32_t row = -1;
        float g = 0.0f;
        if (lane < k) {
            const int32_t sl = slot[t * k + lane];
            const int32_t e = topk_idx[t * k + lane];
            if (sl >= 0 && e >= 0 && e < E) {
                row = offsets[e] + sl;
                g = gates[t * k + lane];
            }
        }
        int32_t rj[KMAX];
        float gj[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            rj[j] = __shfl_sync(0xffffffffu, row, j);
            gj[j] = __shfl_sync(0xffffffffu, g, j);
        }
        for (int c0 = 0; c0 < chunks; c0 += 32 * U) {
            Raw raw[KMAX][U];
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (j < k && rj[j] >= 0 && c < chunks)
                        raw[j][u] = Vec<T, VEC>::load_raw(out_rows + static_cast<int64_t>(rj[j]) * d + c * VEC);
                }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c >= chunks) continue;
                float acc[VEC];
#pragma unroll
                for (int v = 0; v < VEC; ++v) acc[v] = 0.0f;
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (j < k && rj[j] >= 0) {
                        float o[VEC];
                        Vec<T, VEC>::widen(raw[j][u], o);
#pragma unroll
                        for (int v = 0; v < VEC; ++v) acc[v] = fmaf(gj[j], o[v], acc[v]);
                    }
                }
                Vec<T, VEC>::store(y + t * d + c * VEC, acc);
            }
        }
    }
}

// MOE_COMBINE_WARP=0 keeps large batches on the per-chunk kernel (for comparisons).
bool warp_combine_enabled() {
    static const bool enabled = [] {
        const char *v = getenv("MOE_COMBINE_WARP");
        return v == nullptr || atoi(v) != 0;
    }();
    return enabled;
}

template <typename T, int VEC>
cudaError_t launch_combine_t(const void *out_rows, const float *parts, int nparts,
                             int64_t part_stride, const int32_t *slot, const int32_t *topk_idx,
                             const int32_t *offsets, const float *gates, int64_t N, int d, int k,
                             int E, void *y, cudaStream_t s, const float *b_down) {
    const int chunks = d / VEC;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int bpt = (chunks + 127) / 128;
    if (N >= 2048 && nparts == 0 && VEC > 1 && k <= 8 && warp_combine_enabled()) {
        int64_t blocks = (N + 7) / 8;  // 8 warps per block, one token per warp and pass
        if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
        const unsigned gb = static_cast<unsigned>(blocks);
        const T *o = static_cast<const T *>(out_rows);
        T *yy = static_cast<T *>(y);
        // KMAX * U = 6-8 loads of 16 bytes in flight per lane
        if (k <= 2)
            return launch_pdl(combine_warp_kernel<T, VEC, 2, 4>, dim3(gb), dim3(256), 0, s, o, slot, topk_idx,
                              offsets, gates, N, d, k, E, yy);
        if (k <= 4)
            return launch_pdl(combine_warp_kernel<T, VEC, 4, 2>, dim3(gb), dim3(256), 0, s, o, slot, topk_idx,
                              offsets, gates, N, d, k, E, yy);
        if (k <= 6)
            return launch_pdl(combine_warp_kernel<T, VEC, 6, 1>, dim3(gb), dim3(256), 0, s, o, slot, topk_idx,
                              offsets, gates, N, d, k, E, yy);
        return launch_pdl(combine_warp_kernel<T, VEC, 8, 1>, dim3(gb), dim3(256), 0, s, o, slot, topk_idx, offsets,
                          gates, N, d, k, E, yy);
    }
    if (N >= 2048 && nparts == 0 && N * bpt <= INT32_MAX) {
        return launch_pdl(combine_token_kernel<T, VEC>, dim3(static_cast<unsigned>(N * bpt)), dim3(128), 0, s,
                          static_cast<const T *>(out_rows), slot, topk_idx, offsets, gates, N, d, k, E, bpt,
                          static_cast<T *>(y));
    }
    const int threads = chunks >= 256 ? 256 : (chunks >= 128 ? 128 : (chunks >= 64 ? 64 : 32));
    int64_t blocks = N;
    if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
    const size_t smem = sizeof(int32_t) * 3 * static_cast<size_t>(k);
    return launch_pdl(combine_kernel<T, VEC>, dim3(static_cast<unsigned>(blocks)), dim3(threads), smem, s,
                      static_cast<const T *>(out_rows), parts, nparts, part_stride, slot, topk_idx, offsets, gates,
                      N, d, k, E, static_cast<T *>(y), b_down);
}

}  // namespace

cudaError_t launch_combine(const void *out_rows, const float *parts, int nparts,
                           int64_t part_stride, const int32_t *slot, const int32_t *topk_idx,
                           const int32_t *offsets, const float *gates, int dt, int64_t N, int d,
                           int k, int E, void *y, cudaStream_t s, const float *b_down) {
    if (N == 0) return cudaSuccess;
    const bool al = (reinterpret_cast<uintptr_t>(y) % 16 == 0) &&
                    (reinterpret_cast<uintptr_t>(out_rows) % 16 == 0) &&
                    (reinterpret_cast<uintptr_t>(parts) % 16 == 0) &&
                    (reinterpret_cast<uintptr_t>(b_down) % 16 == 0);
    if (dt == 1) {
        if (d % 8 == 0 && al)
            return launch_combine_t<__nv_bfloat16, 8>(out_rows, parts, nparts, part_stride, slot,
                                                      topk_idx, offsets, gates, N, d, k, E, y, s, b_down);
        return launch_combine_t<__nv_bfloat16, 1>(out_rows, parts, nparts, part_stride, slot,
                                                  topk_idx, offsets, gates, N, d, k, E, y, s, b_down);
    }
    if (d % 4 == 0 && al)
        return launch_combine_t<float, 4>(out_rows, parts, nparts, part_stride, slot, topk_idx,
                                          offsets, gates, N, d, k, E, y, s, b_down);
    return launch_combine_t<float, 1>(out_rows, parts, nparts, part_stride, slot, topk_idx,
                                      offsets, gates, N, d, k, E, y, s, b_down);
}

}  // namespace moe
