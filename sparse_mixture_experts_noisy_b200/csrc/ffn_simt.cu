// Expert FFN on CUDA cores: grouped GEMM with fp32 accumulation.
//
// "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 8 (z = W_up x),
// STEP 9 (h = max(0, z)), STEP 10 (E(x) = W_down h).
// Used for fp32 storage (tensor-core tf32 would round the inputs to 10
// mantissa bits and miss the fp32 tolerance) and for bf16 shapes whose rows
// are not 16-byte multiples (tensor-memory copies need them).
//
// out[r, n] = act( sum_k A[r, k] * W[e, n, k] + bias[e, n] )  for the rows r of expert e,
// with A and W K-major.  Tiles of 64 rows x 64 outputs; rows are grouped per
// expert using the device-side counts/offsets, so no host synchronisation.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

// act: 0 none, 1 ReLU, 2 GELU (x * Phi(x)); bias [E][Nw] fp32 or null.
template <typename T>
__global__ void __launch_bounds__(256)
simt_gemm_kernel(const T *__restrict__ A, const T *__restrict__ W, const int32_t *__restrict__ offsets,
                 const int32_t *__restrict__ counts, int E, int Nw, int K, T *__restrict__ out,
                 const float *__restrict__ bias, int act) {
    pdl_trigger();
    pdl_wait();
    __shared__ int32_t tile_prefix[257];
    __shared__ float As[TK][TM + 1];
    __shared__ float Ws[TK][TN + 1];
    const int tid = threadIdx.x;
    if (tid == 0) {
        int32_t run = 0;
        for (int e = 0; e < E; ++e) {
            tile_prefix[e] = run;
            run += (counts[e] + TM - 1) / TM;
        }
        tile_prefix[E] = run;
    }
    __syncthreads();
    const int mt = blockIdx.y;
    if (mt >= tile_prefix[E]) return;
    int e = 0;
    while (e + 1 < E && tile_prefix[e + 1] <= mt) ++e;
    const int m_in = (mt - tile_prefix[e]) * TM;
    const int rows_left = counts[e] - m_in;
    const int64_t row0 = static_cast<int64_t>(offsets[e]) + m_in;
    const int n0 = blockIdx.x * TN;
    const T *We = W + static_cast<int64_t>(e) * Nw * K;

    const int tx = tid & 15, ty = tid >> 4;  // 16 x 16 threads, 4 x 4 outputs each
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += TK) {
        for (int i = tid; i < TK * TM; i += 256) {
            const int kk = i % TK, r = i / TK;
            As[kk][r] = (r < rows_left && k0 + kk < K) ? to_f32<T>(A[(row0 + r) * K + k0 + kk]) : 0.0f;
        }
        for (int i = tid; i < TK * TN; i += 256) {
            const int kk = i % TK, n = i / TK;
            Ws[kk][n] = (n0 + n < Nw && k0 + kk < K)
                            ? to_f32<T>(We[static_cast<int64_t>(n0 + n) * K + k0 + kk])
                            : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
        if (r >= rows_left) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= Nw) continue;
            float v = acc[i][j];
            if (bias) v += bias[static_cast<int64_t>(e) * Nw + n];
            if (act == 2) v = 0.5f * v * (1.0f + erff(v * 0.70710678118654752440f));
            else if (act == 1) v = fmaxf(v, 0.0f);
            out[(row0 + r) * Nw + n] = from_f32<T>(v);
        }
    }
}

template <typename T>
cudaError_t launch_simt_ffn_t(const void *xg, const int32_t *offsets, const int32_t *counts,
                              const void *W_up, const void *W_down, int64_t rows, int d, int d_ff,
                              int E, void *out, void *H, cudaStream_t s, int act, const float *b_up,
                              const float *b_down) {
    const int64_t mtiles = (rows + TM - 1) / TM + E;  // upper bound on sum_e ceil(counts[e] / TM)
    if (mtiles > 65535) return cudaErrorInvalidConfiguration;
    dim3 g_up((d_ff + TN - 1) / TN, static_cast<unsigned>(mtiles));
    cudaError_t e = launch_pdl(simt_gemm_kernel<T>, g_up, dim3(256), 0, s, static_cast<const T *>(xg),
                               static_cast<const T *>(W_up), offsets, counts, E, d_ff, d, static_cast<T *>(H), b_up,
                               act);
    if (e != cudaSuccess) return e;
    dim3 g_dn((d + TN - 1) / TN, static_cast<unsigned>(mtiles));
    return launch_pdl(simt_gemm_kernel<T>, g_dn, dim3(256), 0, s, static_cast<const T *>(H),
                      static_cast<const T *>(W_down), offsets, counts, E, d, d_ff, static_cast<T *>(out), b_down, 0);
}

}  // namespace

cudaError_t launch_simt_ffn(const void *xg, const int32_t *offsets, const int32_t *counts,
                            const void *W_up, const void *W_down, int dt, int64_t rows, int d,
                            int d_ff, int E, void *out, void *H, cudaStream_t s, int act,
                            const float *b_up, const float *b_down) {
    if (dt == 1)
        return launch_simt_ffn_t<__nv_bfloat16>(xg, offsets, counts, W_up, W_down, rows, d, d_ff, E,
                                                out, H, s, act, b_up, b_down);
    return launch_simt_ffn_t<float>(xg, offsets, counts, W_up, W_down, rows, d, d_ff, E, out, H, s, act,
                                    b_up, b_down);
}

}  // namespace moe
