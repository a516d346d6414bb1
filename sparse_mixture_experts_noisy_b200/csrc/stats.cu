// Per-expert load statistics of one routed batch.
//
// "nanoMoEの深層解剖" slide 14: the router returns used_capacity, each
// expert's rows that survive the capacity cut.  This pass gives, per expert e:
//   load[e]        choices (t, j) that picked e, before the cut
//   used[e]        min(load[e], C)
//   importance[e]  the gates of those choices summed: each gate rounded to the
//                  nearest multiple of 2^-32 (ties to even) and added as a
//                  64-bit integer, so the sum is exact and the same in any
//                  order, then scaled back to a double.
// Pass 1: every block counts its grid-stride share of the choices in shared
// memory (integer atomics), then adds its counts into the workspace.  Pass 2
// (one block) writes the outputs.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

struct StatsAcc {
    unsigned long long mass[kStatsMaxE];
    unsigned int load[kStatsMaxE];
};

__global__ void __launch_bounds__(256)
stats_count_kernel(const int32_t *__restrict__ topk_idx, const float *__restrict__ gates, int64_t Nk, int E,
                   StatsAcc *__restrict__ acc) {
    pdl_trigger();
    pdl_wait();
    __shared__ unsigned long long s_mass[kStatsMaxE];
    __shared__ unsigned int s_load[kStatsMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        s_mass[e] = 0ull;
        s_load[e] = 0u;
    }
    __syncthreads();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < Nk;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int32_t e = topk_idx[i];
        if (e < 0 || e >= E) continue;
        atomicAdd(&s_load[e], 1u);
        if (gates != nullptr) {
            const long long m = __double2ll_rn(static_cast<double>(gates[i]) * 4294967296.0);
            atomicAdd(&s_mass[e], static_cast<unsigned long long>(m));  // two's complement: signed sums
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        if (s_load[e] != 0u) atomicAdd(&acc->load[e], s_load[e]);
        if (s_mass[e] != 0ull) atomicAdd(&acc->mass[e], s_mass[e]);
    }
}

__global__ void __launch_bounds__(256)
stats_finish_kernel(const StatsAcc *__restrict__ acc, int E, int64_t C, int32_t *__restrict__ load,
                    int32_t *__restrict__ used, double *__restrict__ importance) {
    pdl_trigger();
    pdl_wait();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const unsigned int l = acc->load[e];
        load[e] = static_cast<int32_t>(l);
        used[e] = static_cast<int32_t>(static_cast<int64_t>(l) < C ? static_cast<int64_t>(l) : C);
        if (importance != nullptr)
            importance[e] = __ll2double_rn(static_cast<long long>(acc->mass[e])) * (1.0 / 4294967296.0);
    }
}

}  // namespace

size_t stats_ws_bytes() { return align_up(sizeof(StatsAcc), 256); }

cudaError_t launch_load_stats(const int32_t *topk_idx, const float *gates, int64_t N, int E, int k, int64_t C,
                              int32_t *load, int32_t *used, double *importance, void *ws, cudaStream_t s) {
    StatsAcc *acc = static_cast<StatsAcc *>(ws);
    cudaError_t e = cudaMemsetAsync(acc, 0, sizeof(StatsAcc), s);
    if (e != cudaSuccess) return e;
    const int64_t Nk = N * k;
    if (Nk > 0) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        int64_t blocks = (Nk + 255) / 256;
        if (blocks > static_cast<int64_t>(sms) * 4) blocks = static_cast<int64_t>(sms) * 4;
        e = launch_pdl(stats_count_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, topk_idx, gates, Nk,
                       E, acc);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(stats_finish_kernel, dim3(1), dim3(256), 0, s, static_cast<const StatsAcc *>(acc), E, C, load,
                      used, importance);
}

}  // namespace moe
