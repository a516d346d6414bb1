// Host-side launchers shared between the C ABI and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Router (route.cu).  status (nullable) is zeroed by the first block.
cudaError_t launch_route(const void *x, int dt, const float *W_g, const float *b_g,
                         const float *noise, float sigma, int64_t N, int d, int E, int k,
                         float *logits_out, int32_t *topk_idx, float *gates, uint32_t *status,
                         cudaStream_t s);

// Dispatch (dispatch.cu).
int64_t dispatch_blocks(int64_t N);
bool dispatch_single_block(int64_t N, int E, int k);
int dispatch_launches(int64_t N, int E, int k);  // kernels launch_dispatch issues
size_t dispatch_ws_bytes(int64_t N, int E, int k);
cudaError_t launch_dispatch(const int32_t *topk_idx, const void *x, int elem_bytes, int64_t N,
                            int d, int E, int k, int64_t C, int32_t *slot, int32_t *counts,
                            int32_t *offsets, void *x_gathered, void *ws, cudaStream_t s);
cudaError_t launch_gather(const int32_t *topk_idx, const int32_t *slot, const int32_t *offsets,
                          const void *x, int elem_bytes, int64_t N, int d, int k, void *x_gathered,
                          cudaStream_t s);

// Combine (combine.cu).  Either out_rows (dtype rows, nparts == 0) or nparts
// fp32 partial buffers `part_stride` elements apart.
cudaError_t launch_combine(const void *out_rows, const float *parts, int nparts,
                           int64_t part_stride, const int32_t *slot, const int32_t *topk_idx,
                           const int32_t *offsets, const float *gates, int dt, int64_t N, int d,
                           int k, int E, void *y, cudaStream_t s);

// CUDA-core expert FFN (ffn_simt.cu).  H: [rows, d_ff] of dtype.
cudaError_t launch_simt_ffn(const void *xg, const int32_t *offsets, const int32_t *counts,
                            const void *W_up, const void *W_down, int dt, int64_t rows, int d,
                            int d_ff, int E, void *out, void *H, cudaStream_t s);

// Tensor-core expert FFN (gemm_tc.cu).
struct TcPlan {
    bool decode;      // weight rows as the MMA's M (few tokens per expert)
    bool pair;        // prefill on CTA pairs (tcgen05 cta_group::2)
    int splits_down;  // K splits of the down projection (decode only)
};
TcPlan plan_tc_ffn(int64_t rows, int d, int d_ff, int E, int num_sms);
size_t tc_ffn_ws_bytes(int64_t rows, int d, int d_ff, int E, int num_sms);
// H: [rows, d_ff] bf16; parts: splits x [rows, d] fp32 (decode plan only).  With
// combine_reads_parts the decode plan leaves the partials for the combine.
cudaError_t launch_tc_ffn(const void *xg, const int32_t *offsets, const int32_t *counts,
                          const void *W_up, const void *W_down, int64_t rows, int d, int d_ff,
                          int E, void *out, void *H, float *parts, bool combine_reads_parts,
                          uint32_t *status, uint64_t timeout_ns, int num_sms, cudaStream_t s,
                          TcPlan *plan_out);
cudaError_t launch_wait_timeout(uint32_t *status, uint64_t timeout_ns, cudaStream_t s);

}  // namespace moe
