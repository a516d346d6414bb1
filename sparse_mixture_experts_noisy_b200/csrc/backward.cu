// Backward pass of the layer for a given routing: the gradients of
// L = sum(dy * y) with respect to x, the router weights and bias, and the
// expert weights.
//
// "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 6 (the
// -inf mask of KeepTopK leaves the kept experts' softmax differentiable and
// the others' gates at 0) and STEP 11 (g_i E_i(x): the gradient reaches the
// router through the gates); "nanoMoEの深層解剖" slide 10 (the router is
// trained by backpropagation).  The top-k indices and the slots are piecewise
// constant and carry no gradient.  For a kept pair (t, j) of expert e, row
// r = offsets[e] + slot[t][j] of the gathered buffers:
//   dg[t][j]  = dy_t . O_r                    (0 for a dropped pair)
//   ds[t][j]  = g_j (dg_j - sum_l g_l dg_l)   (every chosen pair, dropped ones too)
//   dO_r      = g_j dy_t
//   dZ_r      = (dO_r W_down[e]) * [H_r > 0]
//   dX_r      = dZ_r W_up[e]
//   dW_down[e] = sum_r dO_r^T H_r,   dW_up[e] = sum_r dZ_r^T X_r
//   dx_t      = sum_j kept dX_r + sum_j ds_j W_g[e_j]
//   dW_g[e]   = sum over chosen (t, j) of e of ds_j x_t,  db_g[e] = sum of ds_j
// The noise is added to the scores, so ds is also the gradient of the
// pre-noise logits.
//
// This file holds the per-token and router kernels and the CUDA-core GEMMs
// of fp32 storage; the tensor-core GEMMs of bf16 storage are in gemm_tc.cu.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

// ---------------------------------------------------------------- per token
// One warp per token: the gate gradients (dot products of dy_t with the
// token's expert outputs), the score gradients, and the rows dO = g dy_t.
// Lanes take 16-byte chunks of the row when the row is a whole number of
// chunks (VEC elements), single elements otherwise; the lane partial sums go
// through the same shuffle tree every time, so the result is deterministic.
template <typename T, int VEC>
__global__ void __launch_bounds__(256)
bwd_gate_kernel(const T *__restrict__ dy, const T *__restrict__ O, const int32_t *__restrict__ topk,
                const float *__restrict__ gates, const int32_t *__restrict__ slot,
                const int32_t *__restrict__ offsets, int64_t N, int d, int k, T *__restrict__ dO,
                float *__restrict__ ds) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ float bwd_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *dg = bwd_smem + warp * k;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (t >= N) return;
    const T *dyt = dy + t * d;
    const int nv = d / VEC;
    for (int j = 0; j < k; ++j) {
        const int s = slot[t * k + j];
        float acc = 0.0f;
        if (s >= 0) {
            const int e = topk[t * k + j];
            const int64_t row = static_cast<int64_t>(offsets[e]) + s;
            const T *o = O + row * d;
            T *dor = dO + row * d;
            const float g = gates[t * k + j];
            for (int c = lane; c < nv; c += 32) {
                T a[VEC], b[VEC], w[VEC];
                if constexpr (VEC > 1) {
                    *reinterpret_cast<uint4 *>(a) = reinterpret_cast<const uint4 *>(dyt)[c];
                    *reinterpret_cast<uint4 *>(b) = reinterpret_cast<const uint4 *>(o)[c];
                } else {
                    a[0] = dyt[c];
                    b[0] = o[c];
                }
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    const float fa = to_f32(a[v]);
                    acc += fa * to_f32(b[v]);
                    w[v] = from_f32<T>(g * fa);
                }
                if constexpr (VEC > 1) {
                    reinterpret_cast<uint4 *>(dor)[c] = *reinterpret_cast<uint4 *>(w);
                } else {
                    dor[c] = w[0];
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        }
        if (lane == 0) dg[j] = acc;
    }
    __syncwarp();
    if (lane == 0) {
        float sum = 0.0f;
        for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, __fmul_rn(gates[t * k + j], dg[j]));
        for (int j = 0; j < k; ++j) ds[t * k + j] = __fmul_rn(gates[t * k + j], __fsub_rn(dg[j], sum));
    }
}

// One warp per token: dx_t = sum over kept j of dX rows (in j order, fp32)
// plus sum over chosen j of ds_j W_g[e_j] (in j order), rounded once.
template <typename T>
__global__ void __launch_bounds__(256)
bwd_dx_kernel(const T *__restrict__ dX, const float *__restrict__ ds, const float *__restrict__ W_g,
              const int32_t *__restrict__ topk, const int32_t *__restrict__ slot,
              const int32_t *__restrict__ offsets, int64_t N, int d, int k, T *__restrict__ dx) {
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (t >= N) return;
    for (int i = lane; i < d; i += 32) {
        float acc = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int s = slot[t * k + j];
            if (s < 0) continue;
            const int e = topk[t * k + j];
            acc += to_f32(dX[(static_cast<int64_t>(offsets[e]) + s) * d + i]);
        }
        for (int j = 0; j < k; ++j) {
            const int e = topk[t * k + j];
            acc = fmaf(ds[t * k + j], W_g[static_cast<int64_t>(e) * d + i], acc);
        }
        dx[t * d + i] = from_f32<T>(acc);
    }
}

// Router weight gradient, pass 1: block (p, cb) sums the tokens of chunk p
// for the columns cb*128 .. cb*128+127 of every expert; column d is the bias
// (x = 1).  Each thread owns one column, so the sums need no atomics:
// part[p][e][c] = sum over t in chunk p, chosen j with e_j = e, of ds x_t[c].
template <typename T>
__global__ void __launch_bounds__(128)
bwd_router_part_kernel(const T *__restrict__ x, const float *__restrict__ ds, const int32_t *__restrict__ topk,
                       int64_t N, int d, int E, int k, int64_t chunk, float *__restrict__ part) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ float acc_s[];  // [E][128]
    const int c = blockIdx.y * 128 + threadIdx.x;
    const int p = blockIdx.x;
    for (int e = 0; e < E; ++e) acc_s[e * 128 + threadIdx.x] = 0.0f;
    const int64_t t0 = p * chunk, t1 = min(N, t0 + chunk);
    if (c <= d) {
        for (int64_t t = t0; t < t1; ++t) {
            const float xv = c < d ? to_f32(x[t * d + c]) : 1.0f;
            for (int j = 0; j < k; ++j) {
                const int e = topk[t * k + j];
                float &a = acc_s[e * 128 + threadIdx.x];
                a = fmaf(ds[t * k + j], xv, a);
            }
        }
        const int64_t base = static_cast<int64_t>(p) * E * (d + 1);
        for (int e = 0; e < E; ++e) part[base + static_cast<int64_t>(e) * (d + 1) + c] = acc_s[e * 128 + threadIdx.x];
    }
}

// Pass 2: dW_g[e][c] (c < d) and db_g[e] (c = d) = sum of the chunks' parts in chunk order.
__global__ void __launch_bounds__(256)
bwd_router_sum_kernel(const float *__restrict__ part, int P, int d, int E, float *__restrict__ dW_g,
                      float *__restrict__ db_g) {
    pdl_trigger();
    pdl_wait();
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t per = static_cast<int64_t>(E) * (d + 1);
    if (i >= per) return;
    float acc = 0.0f;
    for (int p = 0; p < P; ++p) acc += part[static_cast<int64_t>(p) * per + i];
    const int e = static_cast<int>(i / (d + 1)), c = static_cast<int>(i % (d + 1));
    if (c < d) dW_g[static_cast<int64_t>(e) * d + c] = acc;
    else db_g[e] = acc;
}

// ---------------------------------------------------------------- CUDA-core GEMMs (fp32 storage)
// 64 x 64 output tiles, 256 threads with 4 x 4 outputs each, K staged through
// shared memory 16 at a time; fp32 accumulation in K order.
constexpr int kST = 64, kSK = 16;

__device__ __forceinline__ int expert_of_row(const int32_t *offsets, int E, int64_t r) {
    int lo = 0, hi = E;  // offsets[lo] <= r < offsets[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (offsets[mid] <= r) lo = mid; else hi = mid;
    }
    return lo;
}

// Row-grouped: D[r][n] = sum_kk A[r][kk] * W[e(r)][kk][n] for the kept rows r
// (W stored [E][K][Nw]: the input-gradient GEMMs dO W_down and dZ W_up).
// mask (nullable, [rows][Nw]): D is multiplied by [mask > 0] (the ReLU).
// A 64-row tile may hold rows of two experts: each thread row uses its own
// expert's weights (read through the cache, not staged).
template <typename T>
__global__ void __launch_bounds__(256)
simt_dgrad_kernel(const T *__restrict__ A, const T *__restrict__ W, const int32_t *__restrict__ offsets, int E,
                  int K, int Nw, const T *__restrict__ mask, T *__restrict__ D) {
    pdl_trigger();
    pdl_wait();
    __shared__ float As[kSK][kST + 1];
    const int64_t rows = offsets[E];
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kST;
    if (r0 >= rows) return;
    const int n0 = blockIdx.x * kST;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    int er[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int64_t r = r0 + ty * 4 + a;
        er[a] = r < rows ? expert_of_row(offsets, E, r) : 0;
    }
    for (int k0 = 0; k0 < K; k0 += kSK) {
        for (int q = threadIdx.x; q < kST * kSK; q += 256) {
            const int rr = q / kSK, kk = q % kSK;
            const int64_t r = r0 + rr;
            As[kk][rr] = (r < rows && k0 + kk < K) ? to_f32(A[r * K + k0 + kk]) : 0.0f;
        }
        __syncthreads();
        for (int kk = 0; kk < kSK && k0 + kk < K; ++kk) {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float av = As[kk][ty * 4 + a];
                const T *w = W + (static_cast<int64_t>(er[a]) * K + k0 + kk) * Nw;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int n = n0 + tx * 4 + b;
                    acc[a][b] += av * (n < Nw ? to_f32(w[n]) : 0.0f);
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int64_t r = r0 + ty * 4 + a;
        if (r >= rows) continue;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int n = n0 + tx * 4 + b;
            if (n >= Nw) continue;
            float v = acc[a][b];
            if (mask != nullptr && !(to_f32(mask[r * Nw + n]) > 0.0f)) v = 0.0f;
            D[r * Nw + n] = from_f32<T>(v);
        }
    }
}

// Weight-grouped: D[e][m][n] = sum over expert e's rows r of P[r][m] * Q[r][n]
// (the weight-gradient GEMMs dO^T H and dZ^T X), fp32 out, zero for an
// expert without rows.
template <typename T>
__global__ void __launch_bounds__(256)
simt_wgrad_kernel(const T *__restrict__ P, const T *__restrict__ Q, const int32_t *__restrict__ offsets,
                  const int32_t *__restrict__ counts, int M, int Nn, float *__restrict__ D) {
    pdl_trigger();
    pdl_wait();
    __shared__ float Ps[kSK][kST + 1];
    __shared__ float Qs[kSK][kST + 1];
    const int e = blockIdx.z;
    const int m0 = blockIdx.y * kST, n0 = blockIdx.x * kST;
    const int64_t off = offsets[e];
    const int cnt = counts[e];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < cnt; k0 += kSK) {
        for (int q = threadIdx.x; q < kST * kSK; q += 256) {
            const int kk = q / kST, c = q % kST;
            const bool kv = k0 + kk < cnt;
            const int64_t r = off + k0 + kk;
            Ps[kk][c] = (kv && m0 + c < M) ? to_f32(P[r * M + m0 + c]) : 0.0f;
            Qs[kk][c] = (kv && n0 + c < Nn) ? to_f32(Q[r * Nn + n0 + c]) : 0.0f;
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < kSK; ++kk) {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float pv = Ps[kk][ty * 4 + a];
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] += pv * Qs[kk][tx * 4 + b];
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int m = m0 + ty * 4 + a;
        if (m >= M) continue;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int n = n0 + tx * 4 + b;
            if (n < Nn) D[(static_cast<int64_t>(e) * M + m) * Nn + n] = acc[a][b];
        }
    }
}

template <typename T>
cudaError_t launch_gate(const void *dy, const void *O, const int32_t *topk, const float *gates, const int32_t *slot,
                        const int32_t *offsets, int64_t N, int d, int k, void *dO, float *ds, cudaStream_t s) {
    constexpr int WPB = 8;
    const size_t smem = sizeof(float) * WPB * k;
    const dim3 grid(static_cast<unsigned>((N + WPB - 1) / WPB));
    constexpr int VEC = 16 / sizeof(T);
    const bool vec = (d % VEC) == 0 && (reinterpret_cast<uintptr_t>(dy) % 16) == 0 &&
                     (reinterpret_cast<uintptr_t>(O) % 16) == 0 && (reinterpret_cast<uintptr_t>(dO) % 16) == 0;
    if (vec)
        return launch_pdl(bwd_gate_kernel<T, VEC>, grid, dim3(32 * WPB), smem, s, static_cast<const T *>(dy),
                          static_cast<const T *>(O), topk, gates, slot, offsets, N, d, k, static_cast<T *>(dO), ds);
    return launch_pdl(bwd_gate_kernel<T, 1>, grid, dim3(32 * WPB), smem, s, static_cast<const T *>(dy),
                      static_cast<const T *>(O), topk, gates, slot, offsets, N, d, k, static_cast<T *>(dO), ds);
}

template <typename T>
cudaError_t launch_simt_bwd_gemms(const BwdArgs &a, const void *dO, void *dZ, void *dX, cudaStream_t s) {
    const T *dOt = static_cast<const T *>(dO);
    T *dZt = static_cast<T *>(dZ);
    T *dXt = static_cast<T *>(dX);
    const unsigned rt = static_cast<unsigned>((a.rows + kST - 1) / kST);
    // dZ = (dO W_down[e]) * [H > 0]:  K = d, Nw = d_ff (W_down is [E][d][d_ff])
    cudaError_t e = launch_pdl(simt_dgrad_kernel<T>, dim3((a.d_ff + kST - 1) / kST, rt), dim3(256), 0, s, dOt,
                               static_cast<const T *>(a.W_down), a.offsets, a.E, a.d, a.d_ff,
                               static_cast<const T *>(a.H), dZt);
    if (e != cudaSuccess) return e;
    // dX = dZ W_up[e]:  K = d_ff, Nw = d (W_up is [E][d_ff][d])
    e = launch_pdl(simt_dgrad_kernel<T>, dim3((a.d + kST - 1) / kST, rt), dim3(256), 0, s,
                   static_cast<const T *>(dZt), static_cast<const T *>(a.W_up), a.offsets, a.E, a.d_ff, a.d,
                   static_cast<const T *>(nullptr), dXt);
    if (e != cudaSuccess) return e;
    // dW_down[e] = dO^T H: [d][d_ff];  dW_up[e] = dZ^T X: [d_ff][d]
    e = launch_pdl(simt_wgrad_kernel<T>, dim3((a.d_ff + kST - 1) / kST, (a.d + kST - 1) / kST, a.E), dim3(256), 0,
                   s, dOt, static_cast<const T *>(a.H), a.offsets, a.counts, a.d, a.d_ff, a.dW_down);
    if (e != cudaSuccess) return e;
    return launch_pdl(simt_wgrad_kernel<T>, dim3((a.d + kST - 1) / kST, (a.d_ff + kST - 1) / kST, a.E), dim3(256),
                      0, s, static_cast<const T *>(dZt), static_cast<const T *>(a.x_gathered), a.offsets, a.counts,
                      a.d_ff, a.d, a.dW_up);
}

template <typename T>
cudaError_t launch_tail(const BwdArgs &a, const void *dX, float *ds, float *part, int P, int64_t chunk,
                        int cblocks, cudaStream_t s) {
    constexpr int WPB = 8;
    cudaError_t e = launch_pdl(bwd_dx_kernel<T>, dim3(static_cast<unsigned>((a.N + WPB - 1) / WPB)), dim3(32 * WPB),
                               0, s, static_cast<const T *>(dX), static_cast<const float *>(ds), a.W_g, a.topk,
                               a.slot, a.offsets, a.N, a.d, a.k, static_cast<T *>(a.dx));
    if (e != cudaSuccess) return e;
    const size_t smem = sizeof(float) * static_cast<size_t>(a.E) * 128;
    auto kern = bwd_router_part_kernel<T>;
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    e = launch_pdl(kern, dim3(P, cblocks), dim3(128), smem, s, static_cast<const T *>(a.x),
                   static_cast<const float *>(ds), a.topk, a.N, a.d, a.E, a.k, chunk, part);
    if (e != cudaSuccess) return e;
    const int64_t per = static_cast<int64_t>(a.E) * (a.d + 1);
    return launch_pdl(bwd_router_sum_kernel, dim3(static_cast<unsigned>((per + 255) / 256)), dim3(256), 0, s,
                      static_cast<const float *>(part), P, a.d, a.E, a.dW_g, a.db_g);
}

// Token chunks of the router-gradient pass: enough blocks for about two per SM.
void router_chunks(int64_t N, int d, int num_sms, int &P, int64_t &chunk, int &cblocks) {
    cblocks = (d + 1 + 127) / 128;
    int64_t p = (2 * static_cast<int64_t>(num_sms) + cblocks - 1) / cblocks;
    if (p > N) p = N;
    if (p < 1) p = 1;
    chunk = (N + p - 1) / p;
    P = static_cast<int>((N + chunk - 1) / chunk);
    if (P < 1) P = 1;
}

}  // namespace

BwdLayout bwd_layout(const BwdArgs &a, int num_sms) {
    BwdLayout L{};
    const size_t es = a.dt == 1 ? 2 : 4;
    int P, cblocks;
    int64_t chunk;
    router_chunks(a.N > 0 ? a.N : 1, a.d, num_sms, P, chunk, cblocks);
    size_t o = kStatusBytes;
    L.dO = o; o += align_up(static_cast<size_t>(a.rows) * a.d * es, 256);
    L.dZ = o; o += align_up(static_cast<size_t>(a.rows) * a.d_ff * es, 256);
    L.dX = o; o += align_up(static_cast<size_t>(a.rows) * a.d * es, 256);
    L.ds = o; o += align_up(static_cast<size_t>(a.N) * a.k * 4, 256);
    L.part = o; o += align_up(static_cast<size_t>(P) * a.E * (a.d + 1) * 4, 256);
    L.total = o;
    return L;
}

cudaError_t launch_backward(const BwdArgs &a, void *ws, uint32_t *status, uint64_t timeout_ns, int num_sms,
                            bool tensor_cores, cudaStream_t s) {
    uint8_t *w = static_cast<uint8_t *>(ws);
    const BwdLayout L = bwd_layout(a, num_sms);
    void *dO = w + L.dO, *dZ = w + L.dZ, *dX = w + L.dX;
    float *ds = reinterpret_cast<float *>(w + L.ds);
    float *part = reinterpret_cast<float *>(w + L.part);
    cudaError_t e;
    if (a.N == 0) {
        // no tokens: every gradient is zero
        e = cudaMemsetAsync(a.dW_g, 0, sizeof(float) * a.E * a.d, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.db_g, 0, sizeof(float) * a.E, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.dW_up, 0, sizeof(float) * a.E * a.d_ff * a.d, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.dW_down, 0, sizeof(float) * a.E * a.d * a.d_ff, s);
        return e;
    }
    e = a.dt == 1 ? launch_gate<__nv_bfloat16>(a.dy, a.out_gathered, a.topk, a.gates, a.slot, a.offsets, a.N, a.d,
                                              a.k, dO, ds, s)
                  : launch_gate<float>(a.dy, a.out_gathered, a.topk, a.gates, a.slot, a.offsets, a.N, a.d, a.k, dO,
                                       ds, s);
    if (e != cudaSuccess) return e;
    if (tensor_cores) {
        e = launch_tc_bwd_gemms(a, dO, dZ, dX, status, timeout_ns, num_sms, s);
    } else {
        e = a.dt == 1 ? launch_simt_bwd_gemms<__nv_bfloat16>(a, dO, dZ, dX, s)
                      : launch_simt_bwd_gemms<float>(a, dO, dZ, dX, s);
    }
    if (e != cudaSuccess) return e;
    int P, cblocks;
    int64_t chunk;
    router_chunks(a.N, a.d, num_sms, P, chunk, cblocks);
    return a.dt == 1 ? launch_tail<__nv_bfloat16>(a, dX, ds, part, P, chunk, cblocks, s)
                     : launch_tail<float>(a, dX, ds, part, P, chunk, cblocks, s);
}

int backward_launches(const BwdArgs &a, bool tensor_cores) {
    if (a.N == 0) return 0;
    return 1 + 4 + 3 + (tensor_cores ? 0 : 0);
}

}  // namespace moe
