// Router: logits, noise, KeepTopK and softmax over the kept scores.
//
// "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 2 (s_raw = W_g x),
// STEP 4 (s = s_raw + eps), STEP 5 (-inf outside the top k), STEP 6 (softmax);
// "nanoMoEの深層解剖" slides 11-13 (router in fp32 with autocast disabled, topk,
// -inf scatter, softmax).
//
// One warp owns TPW tokens.  Its lanes split the model dimension d, each lane
// accumulating TPW x 8 partial dot products in fp32 registers (8 experts at a
// time, so x is reused across experts and W_g across tokens), then the warp
// reduces them with shuffles.  The scores of a token then sit in shared memory
// and the warp runs k rounds of a (score desc, index asc) arg-max to pick the
// kept experts; one lane forms the softmax over the k kept scores.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kRouteWarps = 8;
constexpr int kTPW = 4;        // tokens per warp
constexpr int kEC = 8;         // experts per accumulation pass

template <typename T, int VEC>
struct XLoad;
template <>
struct XLoad<__nv_bfloat16, 8> {
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
};
template <>
struct XLoad<float, 4> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[4]) {
        float4 u = *reinterpret_cast<const float4 *>(p);
        v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
    }
};
template <typename T>
struct XLoad<T, 1> {
    static __device__ __forceinline__ void load(const T *p, float (&v)[1]) { v[0] = to_f32<T>(*p); }
};

template <int VEC>
__device__ __forceinline__ void load_w(const float *p, float (&w)[VEC]) {
    if constexpr (VEC == 8) {
        float4 a = *reinterpret_cast<const float4 *>(p);
        float4 b = *reinterpret_cast<const float4 *>(p + 4);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else if constexpr (VEC == 4) {
        float4 a = *reinterpret_cast<const float4 *>(p);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    } else {
        w[0] = *p;
    }
}

// (v, e) ranks before (v2, e2) in KeepTopK order: higher score, then lower index.
__device__ __forceinline__ bool ranks_before(float v, int e, float v2, int e2) {
    return v > v2 || (v == v2 && e < e2);
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_kernel(const T *__restrict__ x, const float *__restrict__ W_g, const float *__restrict__ b_g,
             const float *__restrict__ noise, float sigma, int64_t N, int d, int E, int k,
             float *__restrict__ logits_out, int32_t *__restrict__ topk_idx,
             float *__restrict__ gates, uint32_t *__restrict__ status) {
    extern __shared__ float route_smem[];
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *s_sc = route_smem + static_cast<size_t>(warp) * kTPW * E;           // [TPW][E]
    float *pick_v = route_smem + static_cast<size_t>(kRouteWarps) * kTPW * E +  // [k]
                    static_cast<size_t>(warp) * 2 * k;
    int *pick_e = reinterpret_cast<int *>(pick_v + k);                          // [k]

    const int64_t t0 = (static_cast<int64_t>(blockIdx.x) * kRouteWarps + warp) * kTPW;
    if (t0 >= N) return;  // whole warp leaves together
    const int ntok = (N - t0 < kTPW) ? static_cast<int>(N - t0) : kTPW;
    const bool use_noise = (noise != nullptr) && (sigma != 0.0f);

    // ---- logits: fp32 dot products on CUDA cores
    for (int e0 = 0; e0 < E; e0 += kEC) {
        float acc[kTPW][kEC];
#pragma unroll
        for (int a = 0; a < kTPW; ++a)
#pragma unroll
            for (int c = 0; c < kEC; ++c) acc[a][c] = 0.0f;

        for (int i = lane * VEC; i < d; i += 32 * VEC) {
            float xv[kTPW][VEC];
#pragma unroll
            for (int a = 0; a < kTPW; ++a) {
                if (a < ntok) {
                    XLoad<T, VEC>::load(x + (t0 + a) * static_cast<int64_t>(d) + i, xv[a]);
                } else {
#pragma unroll
                    for (int v = 0; v < VEC; ++v) xv[a][v] = 0.0f;
                }
            }
#pragma unroll
            for (int c = 0; c < kEC; ++c) {
                if (e0 + c < E) {
                    float w[VEC];
                    load_w<VEC>(W_g + static_cast<int64_t>(e0 + c) * d + i, w);
#pragma unroll
                    for (int a = 0; a < kTPW; ++a)
#pragma unroll
                        for (int v = 0; v < VEC; ++v) acc[a][c] = fmaf(xv[a][v], w[v], acc[a][c]);
                }
            }
        }
#pragma unroll
        for (int a = 0; a < kTPW; ++a)
#pragma unroll
            for (int c = 0; c < kEC; ++c) {
                float v = acc[a][c];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                acc[a][c] = v;
            }
        if (lane == 0) {
#pragma unroll
            for (int a = 0; a < kTPW; ++a)
#pragma unroll
                for (int c = 0; c < kEC; ++c)
                    if (e0 + c < E) {
                        float s = acc[a][c];
                        if (b_g) s = __fadd_rn(s, b_g[e0 + c]);
                        s_sc[a * E + e0 + c] = s;
                    }
        }
    }
    __syncwarp();

    // ---- noise, KeepTopK, softmax, one token at a time
    for (int a = 0; a < ntok; ++a) {
        const int64_t t = t0 + a;
        float *sc = s_sc + a * E;
        for (int e = lane; e < E; e += 32) {
            float s = sc[e];
            if (logits_out) logits_out[t * E + e] = s;
            if (use_noise) {
                // two roundings, never fused: fl32(s_raw + fl32(sigma * eps))
                s = __fadd_rn(s, __fmul_rn(sigma, noise[t * E + e]));
                sc[e] = s;
            }
        }
        __syncwarp();
        // previous pick (pv, pe): candidates must rank strictly after it
        float pv = 0.0f;
        int pe = -1;
        for (int j = 0; j < k; ++j) {
            float bv = 0.0f;
            int be = -1;
            for (int e = lane; e < E; e += 32) {
                const float v = sc[e];
                const bool after_prev = (pe < 0) || ranks_before(pv, pe, v, e);
                if (after_prev && (be < 0 || ranks_before(v, e, bv, be))) {
                    bv = v;
                    be = e;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                if (oe >= 0 && (be < 0 || ranks_before(ov, oe, bv, be))) {
                    bv = ov;
                    be = oe;
                }
            }
            if (lane == 0) {
                pick_v[j] = bv;
                pick_e[j] = be;
            }
            pv = bv;
            pe = be;
        }
        __syncwarp();
        if (lane == 0) {
            const float m = pick_v[0];
            float sum = 0.0f;
            for (int j = 0; j < k; ++j) {
                const float ex = expf(__fsub_rn(pick_v[j], m));
                pick_v[j] = ex;
                sum = __fadd_rn(sum, ex);
            }
            for (int j = 0; j < k; ++j) {
                topk_idx[t * k + j] = pick_e[j];
                gates[t * k + j] = __fdiv_rn(pick_v[j], sum);
            }
        }
        __syncwarp();
    }
}

template <typename T, int VEC>
cudaError_t launch_route_t(const void *x, const float *W_g, const float *b_g, const float *noise,
                           float sigma, int64_t N, int d, int E, int k, float *logits_out,
                           int32_t *topk_idx, float *gates, uint32_t *status, cudaStream_t s) {
    const int64_t tok_per_block = kRouteWarps * kTPW;
    const int64_t blocks = (N + tok_per_block - 1) / tok_per_block;
    const size_t smem =
        sizeof(float) * (static_cast<size_t>(kRouteWarps) * kTPW * E + static_cast<size_t>(kRouteWarps) * 2 * k);
    auto kern = route_kernel<T, VEC>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    kern<<<static_cast<unsigned>(blocks), kRouteWarps * 32, smem, s>>>(
        static_cast<const T *>(x), W_g, b_g, noise, sigma, N, d, E, k, logits_out, topk_idx, gates,
        status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const void *x, int dt, const float *W_g, const float *b_g,
                         const float *noise, float sigma, int64_t N, int d, int E, int k,
                         float *logits_out, int32_t *topk_idx, float *gates, uint32_t *status,
                         cudaStream_t s) {
    if (N == 0) return status ? cudaMemsetAsync(status, 0, sizeof(uint32_t), s) : cudaSuccess;
    const uintptr_t ax = reinterpret_cast<uintptr_t>(x), aw = reinterpret_cast<uintptr_t>(W_g);
    if (dt == 1) {
        if (d % 8 == 0 && ax % 16 == 0 && aw % 16 == 0)
            return launch_route_t<__nv_bfloat16, 8>(x, W_g, b_g, noise, sigma, N, d, E, k,
                                                    logits_out, topk_idx, gates, status, s);
        return launch_route_t<__nv_bfloat16, 1>(x, W_g, b_g, noise, sigma, N, d, E, k, logits_out,
                                                topk_idx, gates, status, s);
    }
    if (d % 4 == 0 && ax % 16 == 0 && aw % 16 == 0)
        return launch_route_t<float, 4>(x, W_g, b_g, noise, sigma, N, d, E, k, logits_out,
                                        topk_idx, gates, status, s);
    return launch_route_t<float, 1>(x, W_g, b_g, noise, sigma, N, d, E, k, logits_out, topk_idx,
                                    gates, status, s);
}

}  // namespace moe
