// Capacity-limited dispatch: queue places, drops and the gathered expert batches.
//
// "nanoMoEの深層解剖" slides 14-23: exp_mask = one_hot(topk) permuted to
// [k, tokens, E], cumsum over (k, tokens) - 1 gives each assignment its place in
// its expert's queue (every first choice before every second choice, tokens in
// order within a choice rank), places >= capacity are dropped, used_capacity
// counts the kept ones.  Slides 33-36: the kept tokens are copied into one
// buffer per expert.  The dense one-hot cumsum of the slides is replaced by
// three passes whose result is the same number:
//   1. hist:   per block of kDispatchTB tokens, per choice j, per expert e, the
//              number of (t, j) in the block that chose e;
//   2. scan:   for each (j, e), an exclusive prefix over blocks (in place) and
//              the total over all tokens;
//   3. assign: place(t, j) = sum_{j' < j} total[j'][e] + prefix over earlier
//              blocks + rank among earlier tokens of the same block (warp
//              match + per-warp counts), then slot = place < C ? place : -1;
//   4. gather: the kept rows are copied to x_gathered[offsets[e] + place].
// Batches of at most 1024 tokens do passes 1-3 in one block.
// No step depends on the order in which threads or blocks run.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kDispatchTB = 256;               // tokens per block (one per thread)
constexpr int kDispatchWarps = kDispatchTB / 32;

__global__ void __launch_bounds__(kDispatchTB)
hist_kernel(const int32_t *__restrict__ topk_idx, int64_t N, int E, int k,
            int32_t *__restrict__ hist /* [nblk][k][E] */) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ int32_t h_smem[];  // [E]
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kDispatchTB + threadIdx.x;
    for (int j = 0; j < k; ++j) {
        for (int e = threadIdx.x; e < E; e += blockDim.x) h_smem[e] = 0;
        __syncthreads();
        if (t < N) {
            const int e = topk_idx[t * k + j];
            if (e >= 0 && e < E) atomicAdd(&h_smem[e], 1);
        }
        __syncthreads();
        int32_t *dst = hist + (static_cast<int64_t>(blockIdx.x) * k + j) * E;
        for (int e = threadIdx.x; e < E; e += blockDim.x) dst[e] = h_smem[e];
        __syncthreads();
    }
}

// One warp per (j, e): exclusive prefix of hist[b][j][e] over blocks b, in
// place; the total goes to tot[j][e].
__global__ void __launch_bounds__(256)
scan_kernel(int32_t *__restrict__ hist, int nblk, int E, int k, int32_t *__restrict__ tot) {
    pdl_trigger();
    pdl_wait();
    const int pair = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (pair >= k * E) return;
    const int64_t stride = static_cast<int64_t>(k) * E;
    int32_t carry = 0;
    for (int b0 = 0; b0 < nblk; b0 += 32) {
        const int b = b0 + lane;
        const int32_t v = (b < nblk) ? hist[b * stride + pair] : 0;
        int32_t inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += u;
        }
        if (b < nblk) hist[b * stride + pair] = carry + inc - v;
        carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) tot[pair] = carry;
}

// Queue places and drops for one block of kDispatchTB tokens; block 0 also
// publishes counts and offsets.  hist_excl/tot come from the scan.
__global__ void __launch_bounds__(kDispatchTB)
assign_kernel(const int32_t *__restrict__ topk_idx, int64_t N, int E, int k, int64_t C,
              const int32_t *__restrict__ hist_excl /* [nblk][k][E] */,
              const int32_t *__restrict__ tot /* [k][E] */, int32_t *__restrict__ slot,
              int32_t *__restrict__ counts, int32_t *__restrict__ offsets) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ int32_t a_smem[];
    int32_t *warp_cnt = a_smem;                                // [warps][E]
    int32_t *jrun = warp_cnt + kDispatchWarps * E;             // [E]  sum_{j' < j} tot[j'][e]
    int32_t *offs = jrun + E;                                  // [E + 1]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kDispatchTB + tid;

    // kept rows per expert and their exclusive prefix (every block computes the
    // same values from tot; block 0 publishes them)
    for (int e = tid; e < E; e += blockDim.x) {
        int64_t total = 0;
        for (int j = 0; j < k; ++j) total += tot[j * E + e];
        offs[e] = static_cast<int32_t>(total < C ? total : C);
        jrun[e] = 0;
    }
    __syncthreads();
    if (tid == 0) {
        int32_t run = 0;
        for (int e = 0; e < E; ++e) {
            const int32_t c = offs[e];
            offs[e] = run;
            run += c;
            if (blockIdx.x == 0) counts[e] = c;
        }
        offs[E] = run;
        if (blockIdx.x == 0)
            for (int e = 0; e <= E; ++e) offsets[e] = offs[e];
    }
    __syncthreads();

    const unsigned lt_mask = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
        for (int i = tid; i < kDispatchWarps * E; i += blockDim.x) warp_cnt[i] = 0;
        __syncthreads();
        int e = -1;
        if (t < N) {
            e = topk_idx[t * k + j];
            if (e < 0 || e >= E) e = -1;   // an out-of-range expert id is dropped
        }
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank_in_warp = __popc(same & lt_mask);
        if (e >= 0 && rank_in_warp == 0) warp_cnt[warp * E + e] = __popc(same);
        __syncthreads();
        if (e >= 0) {
            int64_t place = static_cast<int64_t>(jrun[e]) +
                            hist_excl[(static_cast<int64_t>(blockIdx.x) * k + j) * E + e] + rank_in_warp;
            for (int w = 0; w < warp; ++w) place += warp_cnt[w * E + e];
            slot[t * k + j] = place < C ? static_cast<int32_t>(place) : -1;
        } else if (t < N) {
            slot[t * k + j] = -1;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += blockDim.x) jrun[ee] += tot[j * E + ee];
        __syncthreads();
    }
}

// A shard of a batch split over several GPUs (contiguous token ranges, in rank
// order).  base[j][e] is the queue place, in the whole batch, of this shard's
// first j-th choice of expert e; it comes from every shard's counts, exchanged
// once (shard_base_kernel).  C is the whole batch's capacity.  A (t, j) is kept
// iff its place in the whole batch, base[j][e] + its place among this shard's
// j-th choices of e, is below C, which is the unsharded rule.  Kept rows are
// numbered per expert inside the shard (choice rank first, then token order),
// so the shard's gathered rows, expert FFN and combine work unchanged.
__global__ void __launch_bounds__(kDispatchTB)
assign_shard_kernel(const int32_t *__restrict__ topk_idx, int64_t N, int E, int k, int64_t C,
                    const int32_t *__restrict__ hist_excl /* [nblk][k][E] */,
                    const int32_t *__restrict__ tot /* [k][E] this shard's totals */,
                    const int32_t *__restrict__ base /* [k][E] */, int32_t *__restrict__ slot,
                    int32_t *__restrict__ counts, int32_t *__restrict__ offsets) {
    extern __shared__ int32_t a_smem[];
    int32_t *warp_cnt = a_smem;                                // [warps][E]
    int32_t *kept_before = warp_cnt + kDispatchWarps * E;      // [E] kept rows of choices < j
    int32_t *offs = kept_before + E;                           // [E + 1]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kDispatchTB + tid;
    auto kept_of = [&](int j, int e) -> int32_t {  // kept j-th choices of e in this shard
        const int64_t room = C - static_cast<int64_t>(base[j * E + e]);
        const int64_t n = tot[j * E + e];
        return static_cast<int32_t>(room <= 0 ? 0 : (room < n ? room : n));
    };
    for (int e = tid; e < E; e += blockDim.x) {
        int32_t total = 0;
        for (int j = 0; j < k; ++j) total += kept_of(j, e);
        offs[e] = total;
        kept_before[e] = 0;
    }
    __syncthreads();
    if (tid == 0) {
        int32_t run = 0;
        for (int e = 0; e < E; ++e) {
            const int32_t c = offs[e];
            offs[e] = run;
            run += c;
            if (blockIdx.x == 0) counts[e] = c;
        }
        offs[E] = run;
        if (blockIdx.x == 0)
            for (int e = 0; e <= E; ++e) offsets[e] = offs[e];
    }
    __syncthreads();
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
        for (int i = tid; i < kDispatchWarps * E; i += blockDim.x) warp_cnt[i] = 0;
        __syncthreads();
        int e = -1;
        if (t < N) {
            e = topk_idx[t * k + j];
            if (e < 0 || e >= E) e = -1;
        }
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank_in_warp = __popc(same & lt_mask);
        if (e >= 0 && rank_in_warp == 0) warp_cnt[warp * E + e] = __popc(same);
        __syncthreads();
        if (e >= 0) {
            int64_t local = static_cast<int64_t>(hist_excl[(static_cast<int64_t>(blockIdx.x) * k + j) * E + e]) +
                            rank_in_warp;
            for (int w = 0; w < warp; ++w) local += warp_cnt[w * E + e];
            const int64_t place = static_cast<int64_t>(base[j * E + e]) + local;
            slot[t * k + j] = place < C ? static_cast<int32_t>(kept_before[e] + local) : -1;
        } else if (t < N) {
            slot[t * k + j] = -1;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += blockDim.x) kept_before[ee] += kept_of(j, ee);
        __syncthreads();
    }
}

// base[j][e] = sum over all shards of the choices j' < j of e, plus the j-th
// choices of e in the shards before `rank`.  One thread per (j, e).
__global__ void shard_base_kernel(const int32_t *__restrict__ all_counts /* [G][k][E] */, int G, int rank,
                                  int E, int k, int32_t *__restrict__ base) {
    const int pair = blockIdx.x * blockDim.x + threadIdx.x;
    if (pair >= k * E) return;
    const int j = pair / E, e = pair % E;
    int64_t b = 0;
    for (int jj = 0; jj < j; ++jj)
        for (int g = 0; g < G; ++g) b += all_counts[(static_cast<int64_t>(g) * k + jj) * E + e];
    for (int g = 0; g < rank; ++g) b += all_counts[(static_cast<int64_t>(g) * k + j) * E + e];
    base[pair] = static_cast<int32_t>(b);
}

// The whole slot assignment for a batch of at most kSmallTB tokens in one
// block: count per (j, e), then place each (t, j) in token order within its
// choice rank (warp match + per-warp counts), as in the multi-block passes.
constexpr int kSmallTB = 1024;
constexpr int kSmallWarps = kSmallTB / 32;

__global__ void __launch_bounds__(kSmallTB)
dispatch_small_kernel(const int32_t *__restrict__ topk_idx, int64_t N, int E, int k, int64_t C,
                      int32_t *__restrict__ slot, int32_t *__restrict__ counts,
                      int32_t *__restrict__ offsets) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ int32_t s_smem[];
    int32_t *tot = s_smem;                         // [k][E]
    int32_t *warp_cnt = tot + k * E;               // [warps][E]
    int32_t *jrun = warp_cnt + kSmallWarps * E;    // [E]
    int32_t *offs = jrun + E;                      // [E + 1]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = tid;
    for (int i = tid; i < k * E; i += blockDim.x) tot[i] = 0;
    __syncthreads();
    if (t < N)
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[t * k + j];
            if (e >= 0 && e < E) atomicAdd(&tot[j * E + e], 1);
        }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        int64_t total = 0;
        for (int j = 0; j < k; ++j) total += tot[j * E + e];
        offs[e] = static_cast<int32_t>(total < C ? total : C);
        jrun[e] = 0;
    }
    __syncthreads();
    if (tid == 0) {
        int32_t run = 0;
        for (int e = 0; e < E; ++e) {
            const int32_t c = offs[e];
            offs[e] = run;
            counts[e] = c;
            offsets[e] = run;
            run += c;
        }
        offs[E] = run;
        offsets[E] = run;
    }
    __syncthreads();
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
        for (int i = tid; i < kSmallWarps * E; i += blockDim.x) warp_cnt[i] = 0;
        __syncthreads();
        int e = -1;
        if (t < N) {
            e = topk_idx[t * k + j];
            if (e < 0 || e >= E) e = -1;
        }
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank_in_warp = __popc(same & lt_mask);
        if (e >= 0 && rank_in_warp == 0) warp_cnt[warp * E + e] = __popc(same);
        __syncthreads();
        if (e >= 0) {
            int64_t place = static_cast<int64_t>(jrun[e]) + rank_in_warp;
            for (int w = 0; w < warp; ++w) place += warp_cnt[w * E + e];
            slot[t * k + j] = place < C ? static_cast<int32_t>(place) : -1;
        } else if (t < N) {
            slot[t * k + j] = -1;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += blockDim.x) jrun[ee] += tot[j * E + ee];
        __syncthreads();
    }
}

// x_gathered[offsets[e] + slot[t][j]] = x[t] for every kept (t, j): one thread
// per (t, j, unit), units being 16 bytes (2 bytes when rows are not 16-byte
// multiples), so even a handful of tokens spreads over the whole GPU.
template <typename U>
__global__ void __launch_bounds__(256)
gather_kernel(const U *__restrict__ x, int64_t units_per_row, const int32_t *__restrict__ topk_idx,
              const int32_t *__restrict__ slot, const int32_t *__restrict__ offsets, int64_t Nk, int k,
              U *__restrict__ xg) {
    pdl_trigger();
    pdl_wait();
    const int64_t total = Nk * units_per_row;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t tj = i / units_per_row;
        const int64_t c = i - tj * units_per_row;
        const int32_t sl = slot[tj];
        if (sl < 0) continue;
        const int64_t row = static_cast<int64_t>(offsets[topk_idx[tj]]) + sl;
        xg[row * units_per_row + c] = x[(tj / k) * units_per_row + c];
    }
}

// Large batches: one warp per token (grid-stride).  The warp reads the
// token's row once, kGatherUnroll 16-byte pieces per lane in flight, and
// writes it to each kept destination row; lanes j < k look the rows up.
constexpr int kGatherUnroll = 8;

__global__ void __launch_bounds__(256)
gather_warp_kernel(const uint4 *__restrict__ x, int units, const int32_t *__restrict__ topk_idx,
                   const int32_t *__restrict__ slot, const int32_t *__restrict__ offsets, int64_t N, int k,
                   uint4 *__restrict__ xg) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t t = w0; t < N; t += nw) {
        int32_t dest = -1;  // lane j < k: gathered row of choice j, or -1 if dropped
        if (lane < k) {
            const int32_t sl = slot[t * k + lane];
            if (sl >= 0) dest = offsets[topk_idx[t * k + lane]] + sl;
        }
        const uint4 *xr = x + t * units;
        for (int c0 = 0; c0 < units; c0 += 32 * kGatherUnroll) {
            uint4 v[kGatherUnroll];
#pragma unroll
            for (int u = 0; u < kGatherUnroll; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < units) v[u] = xr[c];
            }
            for (int j = 0; j < k; ++j) {
                const int32_t dj = __shfl_sync(0xffffffffu, dest, j);
                if (dj < 0) continue;
                uint4 *dr = xg + static_cast<int64_t>(dj) * units;
#pragma unroll
                for (int u = 0; u < kGatherUnroll; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (c < units) dr[c] = v[u];
                }
            }
        }
    }
}

}  // namespace

int64_t dispatch_blocks(int64_t N) { return (N + kDispatchTB - 1) / kDispatchTB; }

bool dispatch_single_block(int64_t N, int E, int k) {
    const size_t small_smem = sizeof(int32_t) * (static_cast<size_t>(k) * E + kSmallWarps * E + E + E + 1);
    return N <= kSmallTB && small_smem <= 48 * 1024;
}

int dispatch_launches(int64_t N, int E, int k) {
    if (N == 0) return 0;
    return dispatch_single_block(N, E, k) ? 2 : 4;
}

size_t dispatch_ws_bytes(int64_t N, int E, int k) {
    const int64_t nblk = dispatch_blocks(N);
    const size_t hist = sizeof(int32_t) * static_cast<size_t>(nblk > 0 ? nblk : 1) * k * E;
    const size_t tot = sizeof(int32_t) * static_cast<size_t>(k) * E;
    return align_up(hist, 256) + align_up(tot, 256);
}

cudaError_t launch_dispatch(const int32_t *topk_idx, const void *x, int elem_bytes, int64_t N,
                            int d, int E, int k, int64_t C, int32_t *slot, int32_t *counts,
                            int32_t *offsets, void *x_gathered, void *ws, cudaStream_t s) {
    if (N == 0) {
        cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s);
        return e;
    }
    const size_t small_smem = sizeof(int32_t) * (static_cast<size_t>(k) * E + kSmallWarps * E + E + E + 1);
    if (dispatch_single_block(N, E, k)) {
        cudaError_t e = launch_pdl(dispatch_small_kernel, dim3(1), dim3(kSmallTB), small_smem, s, topk_idx, N, E, k,
                                   C, slot, counts, offsets);
        if (e != cudaSuccess) return e;
    } else {
        const int64_t nblk = dispatch_blocks(N);
        int32_t *hist = static_cast<int32_t *>(ws);
        int32_t *tot = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) +
                                                   align_up(sizeof(int32_t) * static_cast<size_t>(nblk) * k * E, 256));
        cudaError_t e = launch_pdl(hist_kernel, dim3(static_cast<unsigned>(nblk)), dim3(kDispatchTB),
                                   sizeof(int32_t) * E, s, topk_idx, N, E, k, hist);
        if (e != cudaSuccess) return e;
        const int pairs = k * E;
        const int warps_per_block = 8;
        e = launch_pdl(scan_kernel, dim3((pairs + warps_per_block - 1) / warps_per_block), dim3(warps_per_block * 32),
                       0, s, hist, static_cast<int>(nblk), E, k, tot);
        if (e != cudaSuccess) return e;
        const size_t smem = sizeof(int32_t) * (static_cast<size_t>(kDispatchWarps) * E + E + E + 1);
        e = launch_pdl(assign_kernel, dim3(static_cast<unsigned>(nblk)), dim3(kDispatchTB), smem, s, topk_idx, N, E,
                       k, C, static_cast<const int32_t *>(hist), static_cast<const int32_t *>(tot), slot, counts,
                       offsets);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_gather(topk_idx, slot, offsets, x, elem_bytes, N, d, k, x_gathered, s);
}

cudaError_t launch_shard_count(const int32_t *topk_idx, int64_t N, int E, int k, int32_t *counts_je,
                               void *ws, cudaStream_t s) {
    if (N == 0) return cudaMemsetAsync(counts_je, 0, sizeof(int32_t) * k * E, s);
    const int64_t nblk = dispatch_blocks(N);
    int32_t *hist = static_cast<int32_t *>(ws);
    hist_kernel<<<static_cast<unsigned>(nblk), kDispatchTB, sizeof(int32_t) * E, s>>>(topk_idx, N, E, k, hist);
    const int pairs = k * E;
    scan_kernel<<<(pairs + 7) / 8, 256, 0, s>>>(hist, static_cast<int>(nblk), E, k, counts_je);
    return cudaGetLastError();
}

cudaError_t launch_shard_base(const int32_t *all_counts, int G, int rank, int E, int k, int32_t *base,
                              cudaStream_t s) {
    const int pairs = k * E;
    shard_base_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(all_counts, G, rank, E, k, base);
    return cudaGetLastError();
}

cudaError_t launch_shard_dispatch(const int32_t *topk_idx, const void *x, int elem_bytes, int64_t N, int d,
                                  int E, int k, int64_t C, const int32_t *counts_je, const int32_t *base,
                                  int32_t *slot, int32_t *counts, int32_t *offsets, void *x_gathered,
                                  void *ws, cudaStream_t s) {
    if (N == 0) {
        cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s);
        return e;
    }
    const int64_t nblk = dispatch_blocks(N);
    const size_t smem = sizeof(int32_t) * (static_cast<size_t>(kDispatchWarps) * E + E + E + 1);
    assign_shard_kernel<<<static_cast<unsigned>(nblk), kDispatchTB, smem, s>>>(
        topk_idx, N, E, k, C, static_cast<const int32_t *>(ws), counts_je, base, slot, counts, offsets);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_gather(topk_idx, slot, offsets, x, elem_bytes, N, d, k, x_gathered, s);
}

cudaError_t launch_gather(const int32_t *topk_idx, const int32_t *slot, const int32_t *offsets,
                          const void *x, int elem_bytes, int64_t N, int d, int k, void *x_gathered,
                          cudaStream_t s) {
    const int64_t row_bytes = static_cast<int64_t>(d) * elem_bytes;
    const bool vec16 = (row_bytes % 16 == 0) && (reinterpret_cast<uintptr_t>(x) % 16 == 0) &&
                       (reinterpret_cast<uintptr_t>(x_gathered) % 16 == 0);
    const int64_t Nk = N * k;
    const int64_t units = vec16 ? row_bytes / 16 : row_bytes / 2;
    const int64_t total = Nk * units;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (vec16 && N >= 2048 && k <= 32 && units <= INT32_MAX) {
        int64_t blocks = (N + 7) / 8;  // 8 warps per block, one token per warp and pass
        if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
        return launch_pdl(gather_warp_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                          static_cast<const uint4 *>(x), static_cast<int>(units), topk_idx, slot, offsets, N, k,
                          static_cast<uint4 *>(x_gathered));
    }
    int64_t blocks = (total + 255) / 256;
    if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
    if (blocks < 1) blocks = 1;
    if (vec16)
        return launch_pdl(gather_kernel<uint4>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                          static_cast<const uint4 *>(x), units, topk_idx, slot, offsets, Nk, k,
                          static_cast<uint4 *>(x_gathered));
    return launch_pdl(gather_kernel<uint16_t>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                      static_cast<const uint16_t *>(x), units, topk_idx, slot, offsets, Nk, k,
                      static_cast<uint16_t *>(x_gathered));
}

}  // namespace moe
