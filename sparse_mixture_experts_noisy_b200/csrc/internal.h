// Host-side launchers shared between the C ABI and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch with programmatic dependent launch allowed: the kernel may be
// scheduled while the previous kernel on the stream finishes; it must call
// pdl_wait() before touching anything that kernel produces or reads.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Router (route.cu).  status (nullable): the status word the tensor-core
// router ORs a timeout into (never cleared here); null selects the library's
// own per-device word (route_status_read_clear).  w3 (nullable):
// route_tc_w3_bytes(d, E) of scratch for the tensor-core router.
cudaError_t launch_route(const void *x, int dt, const float *W_g, const float *b_g,
                         const float *noise, float sigma, int64_t N, int d, int E, int k,
                         float *logits_out, int32_t *topk_idx, float *gates, uint32_t *status,
                         cudaStream_t s, void *w3 = nullptr);
// Kernels launch_route issues for 16-byte-aligned x and W_g (1, or 2 with w3
// on the tensor-core path).
// Whether a tensor-core router call with pre-split weights available reads
// them (the persistent form) rather than splitting W_g in-kernel.
bool route_tc_presplit_used(int64_t N, int d, int E, int sms);
int route_launches(int dt, int64_t N, int d, int E, int k, bool with_w3);

// Tensor-core router for bf16 tokens (route_tc.cu): same results contract as
// launch_route (logits within fp32 accumulation error of the exact dot
// products; KeepTopK and softmax identical).  status nullable.  w3 (nullable,
// route_tc_w3_bytes) is scratch for the pre-split router weights: with it the
// call launches a split pass first and the router reads the parts by TMA;
// without it the router splits in-kernel.  Same results either way.
bool route_tc_shape_ok(int64_t N, int d, int E, int k);  // bf16 tokens of this shape can use it
bool route_tc_eligible(const void *x, const float *W_g, int64_t N, int d, int E, int k);
size_t route_tc_w3_bytes(int d, int E);
cudaError_t launch_route_tc(const void *x, const float *W_g, const float *b_g, const float *noise, float sigma,
                            int64_t N, int d, int E, int k, float *logits_out, int32_t *topk_idx, float *gates,
                            uint32_t *status, uint64_t timeout_ns, void *w3, cudaStream_t s);
// Reads and clears (on stream s, then synchronises it) the library's own status
// word of router calls made without one, on the current device.
cudaError_t route_status_read_clear(uint32_t *word, cudaStream_t s);

// Dispatch (dispatch.cu).
int64_t dispatch_blocks(int64_t N);
bool dispatch_single_block(int64_t N, int E, int k);
int dispatch_launches(int64_t N, int E, int k);  // kernels launch_dispatch issues
size_t dispatch_ws_bytes(int64_t N, int E, int k);
cudaError_t launch_dispatch(const int32_t *topk_idx, const void *x, int elem_bytes, int64_t N,
                            int d, int E, int k, int64_t C, int32_t *slot, int32_t *counts,
                            int32_t *offsets, void *x_gathered, void *ws, cudaStream_t s);
// Token-sharded batches (one exchange of per-(choice, expert) counts).
cudaError_t launch_shard_count(const int32_t *topk_idx, int64_t N, int E, int k, int32_t *counts_je,
                               void *ws, cudaStream_t s);
cudaError_t launch_shard_base(const int32_t *all_counts, int G, int rank, int E, int k, int32_t *base,
                              cudaStream_t s);
cudaError_t launch_shard_dispatch(const int32_t *topk_idx, const void *x, int elem_bytes, int64_t N, int d,
                                  int E, int k, int64_t C, const int32_t *counts_je, const int32_t *base,
                                  int32_t *slot, int32_t *counts, int32_t *offsets, void *x_gathered,
                                  void *ws, cudaStream_t s);
cudaError_t launch_gather(const int32_t *topk_idx, const int32_t *slot, const int32_t *offsets,
                          const void *x, int elem_bytes, int64_t N, int d, int k, void *x_gathered,
                          cudaStream_t s);

// Per-expert load statistics (stats.cu): load before the capacity cut, used =
// min(load, C), gate mass in exact units of 2^-32.  E <= kStatsMaxE.
constexpr int kStatsMaxE = 256;
size_t stats_ws_bytes();
cudaError_t launch_load_stats(const int32_t *topk_idx, const float *gates, int64_t N, int E, int k, int64_t C,
                              int32_t *load, int32_t *used, double *importance, void *ws, cudaStream_t s);

// Combine (combine.cu).  Either out_rows (dtype rows, nparts == 0) or nparts
// fp32 partial buffers `part_stride` elements apart.
// b_down (nullable, [E][d]) is added to the summed partials (nparts > 0 only;
// dtype rows already carry it).
cudaError_t launch_combine(const void *out_rows, const float *parts, int nparts,
                           int64_t part_stride, const int32_t *slot, const int32_t *topk_idx,
                           const int32_t *offsets, const float *gates, int dt, int64_t N, int d,
                           int k, int E, void *y, cudaStream_t s, const float *b_down = nullptr);

// CUDA-core expert FFN (ffn_simt.cu).  H: [rows, d_ff] of dtype.
// act: 1 = ReLU, 2 = GELU; b_up [E][d_ff], b_down [E][d] fp32, nullable.
cudaError_t launch_simt_ffn(const void *xg, const int32_t *offsets, const int32_t *counts,
                            const void *W_up, const void *W_down, int dt, int64_t rows, int d,
                            int d_ff, int E, void *out, void *H, cudaStream_t s, int act = 1,
                            const float *b_up = nullptr, const float *b_down = nullptr);

// Tensor-core expert FFN (gemm_tc.cu).
struct TcPlan {
    bool decode;      // weight rows as the MMA's M (few tokens per expert)
    bool pair;        // prefill on CTA pairs (tcgen05 cta_group::2)
    int splits_up;    // K splits of the up projection (decode only; > 1 adds a ReLU-sum pass)
    int splits_down;  // K splits of the down projection (decode only)
};
TcPlan plan_tc_ffn(int64_t rows, int d, int d_ff, int E, int num_sms);
size_t tc_ffn_ws_bytes(int64_t rows, int d, int d_ff, int E, int num_sms);
int tc_ffn_launches(const TcPlan &p, bool combine_reads_parts);
// H: [rows, d_ff] bf16; parts: splits_down x [rows, d] fp32 then, if
// splits_up > 1, splits_up x [rows, d_ff] fp32 (decode plan only).  With
// combine_reads_parts the decode plan leaves the partials for the combine.
cudaError_t launch_tc_ffn(const void *xg, const int32_t *offsets, const int32_t *counts,
                          const void *W_up, const void *W_down, int64_t rows, int d, int d_ff,
                          int E, void *out, void *H, float *parts, bool combine_reads_parts,
                          uint32_t *status, uint64_t timeout_ns, int num_sms, cudaStream_t s,
                          TcPlan *plan_out, int act = 1, const float *b_up = nullptr,
                          const float *b_down = nullptr);
cudaError_t launch_wait_timeout(uint32_t *status, uint64_t timeout_ns, cudaStream_t s);

// The whole layer for at most 64 bf16 tokens in one cooperative launch
// (decode_fused.cu).  Eligible shapes: E <= 16, k <= 32, the decode plan with
// the up projection split over K (splits_up > 1), the tensor-core router.
// scratch: decode_fused_scratch_bytes(); xg [rows][d], H [rows][d_ff],
// parts_dn [s_dn][rows][d] and parts_up [s_up][rows][d_ff] as in the decode
// plan.  Same results as the separate kernels, bit for bit.
bool decode_fused_eligible(const void *x, const float *W_g, int64_t N, int d, int E, int d_ff, int k, int64_t rows,
                           int num_sms);
size_t decode_fused_scratch_bytes(int64_t N, int d, int E);
cudaError_t launch_decode_fused(const void *x, const float *W_g, const float *b_g, const float *noise, float sigma,
                                int64_t N, int d, int E, int d_ff, int k, int64_t C, const void *W_up,
                                const void *W_down, void *y, float *logits_out, int32_t *topk, float *gates,
                                int32_t *slot, int32_t *counts, int32_t *offsets, void *xg, int64_t rows, void *H,
                                float *parts_dn, float *parts_up, int s_up, int s_dn, void *scratch,
                                uint32_t *status, uint64_t timeout_ns, int num_sms, cudaStream_t s);

// Backward (backward.cu, tensor-core GEMMs in gemm_tc.cu).  Pointers as in
// moe_backward (include/moe.h); dt 1 = bf16 storage, 0 = fp32.
struct BwdArgs {
    const void *x;
    int dt;
    const float *W_g;
    const void *W_up, *W_down;
    int64_t N;
    int d, E, d_ff, k;
    int64_t rows;
    const int32_t *topk;
    const float *gates;
    const int32_t *slot, *offsets, *counts;
    const void *x_gathered, *H, *out_gathered, *dy;
    void *dx;
    float *dW_g, *db_g, *dW_up, *dW_down;
};
// Byte offsets inside the backward workspace (after the status word): the
// gradient rows dO [rows][d], dZ [rows][d_ff], dX [rows][d] of the storage
// type, ds [N][k] fp32, and the router-gradient chunk sums.
struct BwdLayout {
    size_t dO, dZ, dX, ds, part, total;
};
BwdLayout bwd_layout(const BwdArgs &a, int num_sms);
cudaError_t launch_backward(const BwdArgs &a, void *ws, uint32_t *status, uint64_t timeout_ns, int num_sms,
                            bool tensor_cores, cudaStream_t s);
// The four expert GEMMs of the backward on the tensor cores (bf16):
// dZ = (dO W_down[e]) * [H > 0], dX = dZ W_up[e] (CTA pairs, weights read
// MN-major) and dW_down = dO^T H, dW_up = dZ^T X (K = the expert's rows).
cudaError_t launch_tc_bwd_gemms(const BwdArgs &a, const void *dO, void *dZ, void *dX, uint32_t *status,
                                uint64_t timeout_ns, int num_sms, cudaStream_t s);
int backward_launches(const BwdArgs &a, bool tensor_cores);

}  // namespace moe
