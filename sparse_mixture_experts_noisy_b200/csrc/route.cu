// Router: logits, noise, KeepTopK and softmax over the kept scores.
//
// "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 2 (s_raw = W_g x),
// STEP 4 (s = s_raw + eps), STEP 5 (-inf outside the top k), STEP 6 (softmax);
// "nanoMoEの深層解剖" slides 11-13 (router in fp32 with autocast disabled, topk,
// -inf scatter, softmax).
//
// The dot products run on CUDA cores in fp32 (fmaf).  Two launch shapes:
// large batches give one token to each lane (W_g loads are then warp-wide
// broadcasts, registers stay few and occupancy high), small batches give one
// token to a whole block so that even 64 tokens spread over the GPU.  The bias
// and the noise are added with explicit round-to-nearest adds and multiplies,
// so the compiler cannot fuse the noise step into one rounding.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kEC = 8;                  // experts per accumulation pass (small batches)
constexpr int64_t kRouteBlockMaxN = 1024; // up to this many tokens: one block per token

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

// Noise on the fp32 scores of one token (two roundings, never fused):
// s = fl32(s_raw + fl32(sigma * eps)).
__device__ __forceinline__ float add_noise(float s, float sigma, float eps) {
    return __fadd_rn(s, __fmul_rn(sigma, eps));
}

// ------------------------------------------------------------------ large batches
// Lane = token: a block of 4 warps owns 32 tokens; warp w adds up the products of
// its quarter of d, lane by lane, while every lane of the warp reads the same
// W_g entries (broadcast loads that L1 serves once per warp).  The four partial
// sums of a (token, expert) are added in warp order through shared memory.
// Each lane then picks its token's k experts over the E scores and forms the
// softmax.
constexpr int kLaneWarps = 4;

template <typename T, int VEC, int EC>
__global__ void __launch_bounds__(kLaneWarps * 32)
route_lanes_kernel(const T *__restrict__ x, const float *__restrict__ W_g,
                   const float *__restrict__ b_g, const float *__restrict__ noise, float sigma,
                   int64_t N, int d, int E, int k, float *__restrict__ logits_out,
                   int32_t *__restrict__ topk_idx, float *__restrict__ gates,
                   uint32_t *__restrict__ status) {
    extern __shared__ float route_smem[];
    float *part = route_smem;                          // [4 warps][32 lanes][EC + 1]
    float *sc = part + kLaneWarps * 32 * (EC + 1);     // [32 lanes][E + 1]
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * 32 + lane;
    const bool live = t < N;
    const int steps = (d + VEC - 1) / VEC;
    const int i_lo = static_cast<int>(static_cast<int64_t>(warp) * steps / kLaneWarps) * VEC;
    const int i_hi = min(d, static_cast<int>(static_cast<int64_t>(warp + 1) * steps / kLaneWarps) * VEC);
    const T *xr = x + (live ? t : 0) * static_cast<int64_t>(d);

    for (int e0 = 0; e0 < E; e0 += EC) {
        float acc[EC];
#pragma unroll
        for (int c = 0; c < EC; ++c) acc[c] = 0.0f;
        if (live) {
            for (int i = i_lo; i < i_hi; i += VEC) {
                float xv[VEC];
                XLoad<T, VEC>::load(xr + i, xv);
#pragma unroll
                for (int c = 0; c < EC; ++c) {
                    if (e0 + c < E) {
                        float w[VEC];
                        load_w<VEC>(W_g + static_cast<int64_t>(e0 + c) * d + i, w);
#pragma unroll
                        for (int v = 0; v < VEC; ++v) acc[c] = fmaf(xv[v], w[v], acc[c]);
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < EC; ++c) part[(warp * 32 + lane) * (EC + 1) + c] = acc[c];
        __syncthreads();
        if (warp == 0 && live) {
#pragma unroll
            for (int c = 0; c < EC; ++c) {
                if (e0 + c < E) {
                    float v = part[lane * (EC + 1) + c];
#pragma unroll
                    for (int w = 1; w < kLaneWarps; ++w) v = __fadd_rn(v, part[(w * 32 + lane) * (EC + 1) + c]);
                    if (b_g) v = __fadd_rn(v, b_g[e0 + c]);
                    sc[lane * (E + 1) + e0 + c] = v;
                }
            }
        }
        __syncthreads();
    }
    if (warp != 0 || !live) return;

    float *s = sc + lane * (E + 1);
    const bool use_noise = (noise != nullptr) && (sigma != 0.0f);
    for (int e = 0; e < E; ++e) {
        if (logits_out) logits_out[t * E + e] = s[e];
        if (use_noise) s[e] = add_noise(s[e], sigma, noise[t * E + e]);
    }
    // k picks in (score desc, index asc) order; softmax shifted by the first pick
    float pv = 0.0f, m = 0.0f, sum = 0.0f;
    int pe = -1;
    for (int j = 0; j < k; ++j) {
        float bv = 0.0f;
        int be = -1;
        for (int e = 0; e < E; ++e) {
            const float v = s[e];
            if ((pe < 0 || ranks_before(pv, pe, v, e)) && (be < 0 || ranks_before(v, e, bv, be))) {
                bv = v;
                be = e;
            }
        }
        if (j == 0) m = bv;
        sum = __fadd_rn(sum, expf(__fsub_rn(bv, m)));
        topk_idx[t * k + j] = be;
        pv = bv;
        pe = be;
    }
    for (int j = 0; j < k; ++j) {
        const float v = s[topk_idx[t * k + j]];
        gates[t * k + j] = __fdiv_rn(expf(__fsub_rn(v, m)), sum);
    }
}

// ------------------------------------------------------------------ small batches
// One token per block: the 128 threads split d, each keeps 8 experts' partial
// sums, the block adds them (shuffles, then the 4 warps in order), and warp 0
// runs k rounds of a warp-wide (score desc, index asc) arg-max and the softmax.
template <typename T, int VEC>
__global__ void __launch_bounds__(128)
route_block_kernel(const T *__restrict__ x, const float *__restrict__ W_g,
                   const float *__restrict__ b_g, const float *__restrict__ noise, float sigma,
                   int64_t N, int d, int E, int k, float *__restrict__ logits_out,
                   int32_t *__restrict__ topk_idx, float *__restrict__ gates,
                   uint32_t *__restrict__ status) {
    extern __shared__ float route_smem[];
    float *part = route_smem;          // [4 warps][kEC]
    float *sc = part + 4 * kEC;        // [E]
    float *pick_v = sc + E;            // [k]
    int *pick_e = reinterpret_cast<int *>(pick_v + k);  // [k]
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = blockIdx.x;
    const T *xr = x + t * static_cast<int64_t>(d);
    for (int e0 = 0; e0 < E; e0 += kEC) {
        float acc[kEC];
#pragma unroll
        for (int c = 0; c < kEC; ++c) acc[c] = 0.0f;
        for (int i = threadIdx.x * VEC; i < d; i += 128 * VEC) {
            float xv[VEC];
            XLoad<T, VEC>::load(xr + i, xv);
#pragma unroll
            for (int c = 0; c < kEC; ++c) {
                if (e0 + c < E) {
                    float w[VEC];
                    load_w<VEC>(W_g + static_cast<int64_t>(e0 + c) * d + i, w);
#pragma unroll
                    for (int v = 0; v < VEC; ++v) acc[c] = fmaf(xv[v], w[v], acc[c]);
                }
            }
        }
#pragma unroll
        for (int c = 0; c < kEC; ++c) {
            float v = acc[c];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) part[warp * kEC + c] = v;
        }
        __syncthreads();
        if (threadIdx.x < kEC && e0 + threadIdx.x < E) {
            const int c = threadIdx.x;
            float v = part[c];
            for (int w = 1; w < 4; ++w) v = __fadd_rn(v, part[w * kEC + c]);
            if (b_g) v = __fadd_rn(v, b_g[e0 + c]);
            sc[e0 + c] = v;
        }
        __syncthreads();
    }
    if (warp != 0) return;
    const bool use_noise = (noise != nullptr) && (sigma != 0.0f);
    for (int e = lane; e < E; e += 32) {
        float v = sc[e];
        if (logits_out) logits_out[t * E + e] = v;
        if (use_noise) sc[e] = add_noise(v, sigma, noise[t * E + e]);
    }
    __syncwarp();
    float pv = 0.0f;
    int pe = -1;
    for (int j = 0; j < k; ++j) {
        float bv = 0.0f;
        int be = -1;
        for (int e = lane; e < E; e += 32) {
            const float v = sc[e];
            if ((pe < 0 || ranks_before(pv, pe, v, e)) && (be < 0 || ranks_before(v, e, bv, be))) {
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
        for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, expf(__fsub_rn(pick_v[j], m)));
        for (int j = 0; j < k; ++j) {
            topk_idx[t * k + j] = pick_e[j];
            gates[t * k + j] = __fdiv_rn(expf(__fsub_rn(pick_v[j], m)), sum);
        }
    }
}

template <typename T, int VEC>
cudaError_t launch_route_v(const void *x, const float *W_g, const float *b_g, const float *noise,
                           float sigma, int64_t N, int d, int E, int k, float *logits_out,
                           int32_t *topk_idx, float *gates, uint32_t *status, cudaStream_t s) {
    const T *xt = static_cast<const T *>(x);
    if (N <= kRouteBlockMaxN) {
        const size_t smem = sizeof(float) * (4 * kEC + E + 2 * static_cast<size_t>(k));
        route_block_kernel<T, VEC><<<static_cast<unsigned>(N), 128, smem, s>>>(
            xt, W_g, b_g, noise, sigma, N, d, E, k, logits_out, topk_idx, gates, status);
        return cudaGetLastError();
    }
    const int64_t blocks = (N + 31) / 32;
    if (E <= 8) {
        const size_t smem = sizeof(float) * (kLaneWarps * 32 * (8 + 1) + 32 * (E + 1));
        route_lanes_kernel<T, VEC, 8><<<static_cast<unsigned>(blocks), kLaneWarps * 32, smem, s>>>(
            xt, W_g, b_g, noise, sigma, N, d, E, k, logits_out, topk_idx, gates, status);
    } else {
        const size_t smem = sizeof(float) * (kLaneWarps * 32 * (16 + 1) + 32 * (E + 1));
        route_lanes_kernel<T, VEC, 16><<<static_cast<unsigned>(blocks), kLaneWarps * 32, smem, s>>>(
            xt, W_g, b_g, noise, sigma, N, d, E, k, logits_out, topk_idx, gates, status);
    }
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
            return launch_route_v<__nv_bfloat16, 8>(x, W_g, b_g, noise, sigma, N, d, E, k,
                                                    logits_out, topk_idx, gates, status, s);
        return launch_route_v<__nv_bfloat16, 1>(x, W_g, b_g, noise, sigma, N, d, E, k, logits_out,
                                                topk_idx, gates, status, s);
    }
    if (d % 4 == 0 && ax % 16 == 0 && aw % 16 == 0)
        return launch_route_v<float, 4>(x, W_g, b_g, noise, sigma, N, d, E, k, logits_out,
                                        topk_idx, gates, status, s);
    return launch_route_v<float, 1>(x, W_g, b_g, noise, sigma, N, d, E, k, logits_out, topk_idx,
                                    gates, status, s);
}

}  // namespace moe
