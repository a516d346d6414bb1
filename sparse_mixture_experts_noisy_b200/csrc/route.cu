// Router: logits, noise, KeepTopK and softmax over the kept scores.
//
// "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 2 (s_raw = W_g x),
// STEP 4 (s = s_raw + eps), STEP 5 (-inf outside the top k), STEP 6 (softmax);
// "nanoMoEの深層解剖" slides 11-13 (router in fp32 with autocast disabled, topk,
// -inf scatter, softmax).
//
// bf16 tokens with d a multiple of 8, at most 160 experts and k <= 32 route on the
// tensor cores (route_tc.cu).  Everything else runs here, on CUDA cores in
// fp32 (fmaf), in one of two launch shapes: large batches give 4 tokens to
// each warp with W_g staged in shared memory, small batches give one token to
// a whole block.  Both sum every dot product in the same order, so the choice
// between them never changes a result.  The bias and the noise are added with
// explicit round-to-nearest adds and multiplies, so the compiler cannot fuse
// the noise step into one rounding.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kEC = 8;                  // experts per accumulation pass (small batches)
constexpr int64_t kRouteBlockMaxN = 1024; // up to this many tokens: one block per token
constexpr uint64_t kRouteWaitTimeoutNs = 1000000000ull;  // tensor-core router: 1 s per wait

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
// A block of 8 warps owns 32 tokens, 4 per warp.  For each 1024-wide chunk of
// d the block stages W_g[e0 .. e0+8)[chunk] in shared memory; the lanes of a
// warp read 16-byte pieces of their 4 tokens' rows (consecutive lanes,
// consecutive bytes) and keep 4 tokens x 8 experts of fp32 partial sums, which
// the warp adds with shuffles once d is done.  Then the warp picks each
// token's k experts (rounds of a warp-wide arg-max) and forms the softmax.
constexpr int kTileWarps = 8;
constexpr int kTileTPW = 4;                    // tokens per warp
constexpr int kTileTok = kTileWarps * kTileTPW;
constexpr int kTileDC = 1024;                  // d chunk staged per pass
constexpr int kTileEC = 8;                     // experts per pass

template <typename T, int VEC>
__global__ void __launch_bounds__(kTileWarps * 32)
route_tile_kernel(const T *__restrict__ x, const float *__restrict__ W_g,
                  const float *__restrict__ b_g, const float *__restrict__ noise, float sigma,
                  int64_t N, int d, int E, int k, float *__restrict__ logits_out,
                  int32_t *__restrict__ topk_idx, float *__restrict__ gates,
                  uint32_t *__restrict__ status) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ float route_smem[];
    float *ws = route_smem;                               // [kTileEC][kTileDC]
    float *s_sc = ws + kTileEC * kTileDC;                  // [kTileTok][E]
    float *pick_v = s_sc + static_cast<size_t>(kTileTok) * E + static_cast<size_t>(threadIdx.x >> 5) * 2 * k;
    int *pick_e = reinterpret_cast<int *>(pick_v + k);
    (void)status;  // no waits here, so nothing to report
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTileTok + warp * kTileTPW;
    const int ntok = (t0 >= N) ? 0 : ((N - t0 < kTileTPW) ? static_cast<int>(N - t0) : kTileTPW);
    const bool vec_w = (d % 4 == 0) && (reinterpret_cast<uintptr_t>(W_g) % 16 == 0);

    for (int e0 = 0; e0 < E; e0 += kTileEC) {
        float acc[kTileTPW][kTileEC];
#pragma unroll
        for (int a = 0; a < kTileTPW; ++a)
#pragma unroll
            for (int c = 0; c < kTileEC; ++c) acc[a][c] = 0.0f;
        for (int dc = 0; dc < d; dc += kTileDC) {
            const int dn = min(kTileDC, d - dc);
            __syncthreads();
            if (vec_w) {
                // 16-byte pieces, every one of the thread's loads in flight at once
                constexpr int kPieces = kTileEC * kTileDC / 4 / (kTileWarps * 32);
                float4 tmp[kPieces];
#pragma unroll
                for (int u = 0; u < kPieces; ++u) {
                    const int i = (threadIdx.x + u * kTileWarps * 32) * 4;
                    const int c = i / kTileDC, j = i % kTileDC;
                    tmp[u] = (e0 + c < E && j < dn)
                                 ? *reinterpret_cast<const float4 *>(W_g + static_cast<int64_t>(e0 + c) * d + dc + j)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u = 0; u < kPieces; ++u)
                    reinterpret_cast<float4 *>(ws)[threadIdx.x + u * kTileWarps * 32] = tmp[u];
            } else {
                for (int i = threadIdx.x; i < kTileEC * kTileDC; i += blockDim.x) {
                    const int c = i / kTileDC, j = i % kTileDC;
                    ws[i] = (e0 + c < E && j < dn) ? W_g[static_cast<int64_t>(e0 + c) * d + dc + j] : 0.0f;
                }
            }
            __syncthreads();
            if (ntok > 0) {
#pragma unroll 1
                for (int j = lane * VEC; j < dn; j += 32 * VEC) {
                    float xv[kTileTPW][VEC];
#pragma unroll
                    for (int a = 0; a < kTileTPW; ++a) {
                        if (a < ntok) {
                            XLoad<T, VEC>::load(x + (t0 + a) * static_cast<int64_t>(d) + dc + j, xv[a]);
                        } else {
#pragma unroll
                            for (int v = 0; v < VEC; ++v) xv[a][v] = 0.0f;
                        }
                    }
#pragma unroll
                    for (int c = 0; c < kTileEC; ++c) {
                        float w[VEC];
                        load_w<VEC>(ws + c * kTileDC + j, w);
#pragma unroll
                        for (int a = 0; a < kTileTPW; ++a)
#pragma unroll
                            for (int v = 0; v < VEC; ++v) acc[a][c] = fmaf(xv[a][v], w[v], acc[a][c]);
                    }
                }
            }
        }
#pragma unroll
        for (int a = 0; a < kTileTPW; ++a)
#pragma unroll
            for (int c = 0; c < kTileEC; ++c) {
                float v = acc[a][c];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                acc[a][c] = v;
            }
        if (lane == 0) {
#pragma unroll
            for (int a = 0; a < kTileTPW; ++a)
#pragma unroll
                for (int c = 0; c < kTileEC; ++c)
                    if (a < ntok && e0 + c < E) {
                        float v = acc[a][c];
                        if (b_g) v = __fadd_rn(v, b_g[e0 + c]);
                        s_sc[(warp * kTileTPW + a) * E + e0 + c] = v;
                    }
        }
    }
    __syncwarp();
    const bool use_noise = (noise != nullptr) && (sigma != 0.0f);
    for (int a = 0; a < ntok; ++a) {
        const int64_t t = t0 + a;
        float *sc = s_sc + (warp * kTileTPW + a) * E;
        for (int e = lane; e < E; e += 32) {
            const float v = sc[e];
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
        __syncwarp();
    }
}

// ------------------------------------------------------------------ small batches
// One token per block, so that even a few tokens spread over the GPU.  Warp w
// takes experts w, w+4, w+8, ... (kEC of them per pass) and sums each dot
// product exactly as the large-batch kernel does: lane l runs one fmaf chain
// over the VEC-wide pieces l, l+32, l+64, ... of d, then the warp adds the
// lanes with the same xor-shuffle tree.  So a token gets the same logits, bit
// for bit, whatever the batch size.  Warp 0 then runs k rounds of a warp-wide
// (score desc, index asc) arg-max and the softmax.
template <typename T, int VEC>
__global__ void __launch_bounds__(128)
route_block_kernel(const T *__restrict__ x, const float *__restrict__ W_g,
                   const float *__restrict__ b_g, const float *__restrict__ noise, float sigma,
                   int64_t N, int d, int E, int k, float *__restrict__ logits_out,
                   int32_t *__restrict__ topk_idx, float *__restrict__ gates,
                   uint32_t *__restrict__ status) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ float route_smem[];
    float *sc = route_smem;            // [E]
    float *pick_v = sc + E;            // [k]
    int *pick_e = reinterpret_cast<int *>(pick_v + k);  // [k]
    (void)status;  // no waits here, so nothing to report
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = blockIdx.x;
    const T *xr = x + t * static_cast<int64_t>(d);
    for (int g0 = warp; g0 < E; g0 += 4 * kEC) {  // experts g0 + 4c, c < kEC
        float acc[kEC];
#pragma unroll
        for (int c = 0; c < kEC; ++c) acc[c] = 0.0f;
#pragma unroll 1
        for (int j = lane * VEC; j < d; j += 32 * VEC) {
            float xv[VEC];
            XLoad<T, VEC>::load(xr + j, xv);
#pragma unroll
            for (int c = 0; c < kEC; ++c) {
                const int e = g0 + 4 * c;
                if (e < E) {
                    float w[VEC];
                    load_w<VEC>(W_g + static_cast<int64_t>(e) * d + j, w);
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
            const int e = g0 + 4 * c;
            if (lane == 0 && e < E) sc[e] = b_g ? __fadd_rn(v, b_g[e]) : v;
        }
    }
    __syncthreads();
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
        const size_t smem = sizeof(float) * (E + 2 * static_cast<size_t>(k));
        return launch_pdl(route_block_kernel<T, VEC>, dim3(static_cast<unsigned>(N)), dim3(128), smem, s, xt, W_g,
                          b_g, noise, sigma, N, d, E, k, logits_out, topk_idx, gates, status);
    }
    const int64_t blocks = (N + kTileTok - 1) / kTileTok;
    const size_t smem = sizeof(float) * (static_cast<size_t>(kTileEC) * kTileDC +
                                         static_cast<size_t>(kTileTok) * E + static_cast<size_t>(kTileWarps) * 2 * k);
    auto kern = route_tile_kernel<T, VEC>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(kTileWarps * 32), smem, s, xt, W_g, b_g,
                      noise, sigma, N, d, E, k, logits_out, topk_idx, gates, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const void *x, int dt, const float *W_g, const float *b_g,
                         const float *noise, float sigma, int64_t N, int d, int E, int k,
                         float *logits_out, int32_t *topk_idx, float *gates, uint32_t *status,
                         cudaStream_t s, void *w3) {
    if (N == 0) return cudaSuccess;
    const uintptr_t ax = reinterpret_cast<uintptr_t>(x), aw = reinterpret_cast<uintptr_t>(W_g);
    if (dt == 1 && route_tc_eligible(x, W_g, N, d, E, k))
        return launch_route_tc(x, W_g, b_g, noise, sigma, N, d, E, k, logits_out, topk_idx, gates, status,
                               kRouteWaitTimeoutNs, w3, s);
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

int route_launches(int dt, int64_t N, int d, int E, int k, bool with_w3) {
    if (N == 0) return 0;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return (dt == 1 && route_tc_shape_ok(N, d, E, k) && with_w3 && route_tc_presplit_used(N, d, E, sms)) ? 2 : 1;
}

}  // namespace moe
