// Expert FFN on the fifth-generation tensor cores: a persistent grouped GEMM
// with tcgen05.mma (bf16 inputs, fp32 accumulators in tensor memory) fed by
// TMA, one CTA per SM.
//
// "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 8 (z = W_up x),
// STEP 9 (ReLU, fused into the up-projection epilogue), STEP 10 (W_down h);
// "nanoMoEの深層解剖" slide 32 (MLPExperts: one batched matmul per projection
// over all experts).  The slides' bmm over a dense [E, capacity, d] batch is
// replaced by a grouped GEMM over the compact expert-major rows, so padding
// and dropped slots cost nothing.
//
//   D[r, n] = sum_k T[r, k] * W[e, n, k]        r in expert e's rows, n < Nw
//
// T ("token rows": x_gathered or the hidden activations) is [rows, K] and W is
// [E, Nw, K]; both are K-major, which is what tcgen05 reads without transposes.
//
// Two tile orientations:
//   - prefill (SWAP = false): the MMA's M = 128 token rows, N = BN weight rows;
//   - decode  (SWAP = true):  M = 128 weight rows, N = up to BN tokens of one
//     expert, so a 64-token batch still streams each weight tile once through
//     a full-height MMA.
// Work units are (expert, M tile, N tile, K split), enumerated from the
// device-side counts by every CTA identically, and dealt round-robin.
//
// Warp roles (192 threads): warp 0 lane 0 issues TMA loads into a STAGES-deep
// shared-memory ring; warp 1 owns the tensor memory and its lane 0 issues the
// MMAs (4 x K=16 per 64-wide K block) and commits; warps 2-5 drain finished
// accumulators (tcgen05.ld 32x32b: warp w reads TMEM lanes 32*(w%4)..+31),
// apply ReLU, convert and store.  Two accumulator buffers let the epilogue of
// one unit overlap the MMAs of the next.  Every wait is bounded in time: on
// expiry the kernel records ST_TIMEOUT, lets in-flight copies and MMAs land,
// frees its tensor memory and exits.
#include "common.cuh"
#include "internal.h"
#include "tmap.h"

#include <cstdlib>

namespace moe {

namespace {

constexpr int kBM = 128;       // MMA M
constexpr int kBK = 64;        // K elements per stage (128 bytes of bf16 = one swizzle row)
static_assert(kBK == kTmapBoxK, "tensor-map box K");
constexpr int kThreads = 192;

// Epilogues: bf16 out with the optional bias (down projection), bf16 out with
// bias and activation (up projection), raw fp32 partial sums (K splits; bias
// and activation are applied once the splits are added), bf16 out zeroed
// where a mask array is not positive (the ReLU's derivative in the backward).
// bf16 out (+ bias), bf16 out of bias + activation, fp32 partials, bf16 out
// zeroed where a mask is not positive; and two fixed forms of the first two for
// the layer without biases (ReLU only, nothing), whose epilogues carry no
// runtime branches, and so much less code.
enum { EPI_BF16 = 0, EPI_BF16_ACT = 1, EPI_F32 = 2, EPI_BF16_MASK = 3, EPI_BF16_RELU = 4, EPI_BF16_PLAIN = 5 };

struct TcArgs {
    const int32_t *offsets;
    const int32_t *counts;
    int E, Nw, K, splits;
    void *out;
    int64_t ldo;           // elements per output row
    int64_t split_stride;  // elements between K-split partial buffers (EPI_F32)
    uint32_t *status;
    uint64_t timeout_ns;
    const float *bias;  // [E][Nw] fp32 or null: added to every output row of expert e
    int act;            // EPI_BF16_ACT: 1 = ReLU, 2 = GELU (x * Phi(x))
    const __nv_bfloat16 *mask;  // EPI_BF16_MASK: [rows][Nw], same layout as out
};

__device__ __forceinline__ float activate(float v, int act) {
    if (act == 2) return 0.5f * v * (1.0f + erff(v * 0.70710678118654752440f));
    return fmaxf(v, 0.0f);
}

// Bias and activation for one 32-column chunk of TMEM values.  Token-row tiles
// (swap = false): columns are weight rows col0..col0+31, the same for all lanes.
// Weight-row tiles (swap = true): the lane's weight row w is fixed.
template <int EPI, bool SWAP>
__device__ __forceinline__ void bias_act(uint32_t (&r)[32], const TcArgs &args, int e, int col0, int w) {
    if (EPI == EPI_F32 || EPI == EPI_BF16_PLAIN || EPI == EPI_BF16_MASK) return;  // no bias, no activation
    if (EPI == EPI_BF16_RELU) {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(fmaxf(__uint_as_float(r[i]), 0.0f));
        return;
    }
    if (args.bias != nullptr) {
        const float *b = args.bias + static_cast<int64_t>(e) * args.Nw;
        if (SWAP) {
            const float bw = (w < args.Nw) ? b[w] : 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) + bw);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (col0 + i < args.Nw) r[i] = __float_as_uint(__uint_as_float(r[i]) + b[col0 + i]);
        }
    }
    if (EPI == EPI_BF16_ACT) {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(activate(__uint_as_float(r[i]), args.act));
    }
}

template <int BN>
__host__ __device__ constexpr uint32_t tmem_cols() {
    return 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
}

struct Unit {
    int e;
    int tok0;     // first token row of the unit inside expert e
    int w0;       // first weight row of the unit
    int kb0, kb1; // K blocks [kb0, kb1)
    int split;
    int n_valid;  // valid columns of the MMA's N dimension
};

template <int BN, bool SWAP>
__device__ __forceinline__ Unit decode_unit(int u, const int32_t *pre, const int32_t *cnt, int E,
                                            int Nw, int splits, int kb_total) {
    int lo = 0, hi = E;  // pre[lo] <= u < pre[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] <= u) lo = mid; else hi = mid;
    }
    Unit t;
    t.e = lo;
    int r = u - pre[lo];
    t.split = r % splits;
    r /= splits;
    const int c = cnt[lo];
    if (!SWAP) {
        const int mt = (c + kBM - 1) / kBM;
        const int m = r % mt, n = r / mt;
        t.tok0 = m * kBM;
        t.w0 = n * BN;
        t.n_valid = min(BN, Nw - t.w0);
    } else {
        const int tt = (c + BN - 1) / BN;
        const int m = r / tt, n = r % tt;
        t.w0 = m * kBM;
        t.tok0 = n * BN;
        t.n_valid = min(BN, c - t.tok0);
    }
    t.kb0 = static_cast<int>(static_cast<int64_t>(t.split) * kb_total / splits);
    t.kb1 = static_cast<int>(static_cast<int64_t>(t.split + 1) * kb_total / splits);
    return t;
}

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > timeout_ns) return false;
    return true;
}

template <int BN, bool SWAP, int EPI, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_tok, const __grid_constant__ CUtensorMap tm_w,
               const TcArgs args) {
    constexpr uint32_t A_BYTES = kBM * kBK * 2;
    constexpr uint32_t B_BYTES = BN * kBK * 2;
    constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    constexpr uint32_t TMEM_COLS = tmem_cols<BN>();
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN");
    static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");

    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t bars[2 * STAGES + 5];
    __shared__ uint32_t tmem_holder;
    __shared__ int32_t pre_s[257];
    __shared__ int32_t cnt_s[256];
    __shared__ uint32_t cta_status;  // this CTA's copy of the status word

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = args.E, Nw = args.Nw, splits = args.splits;
    const int kb_total = (args.K + kBK - 1) / kBK;
    uint32_t *status = &cta_status;
    const uint64_t tmo = args.timeout_ns;

    const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    const uint32_t full0 = smem_u32(&bars[0]);
    const uint32_t empty0 = smem_u32(&bars[STAGES]);
    const uint32_t tfull0 = smem_u32(&bars[2 * STAGES]);
    const uint32_t tempty0 = smem_u32(&bars[2 * STAGES + 2]);
    const uint32_t drain = smem_u32(&bars[2 * STAGES + 4]);

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(tfull0, 1);
        mbar_init(tfull0 + 8, 1);
        mbar_init(tempty0, 4);
        mbar_init(tempty0 + 8, 4);
        mbar_init(drain, 1);
        fence_barrier_init();
        cta_status = 0u;
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_tok);
        tma_prefetch_desc(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tmem_holder), TMEM_COLS);
        tmem_relinquish();
    }
    pdl_wait();
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt_s[e] = args.counts[e];
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            pre_s[e] = run;
            const int c = cnt_s[e];
            const int units = SWAP ? ((Nw + kBM - 1) / kBM) * ((c + BN - 1) / BN)
                                   : ((c + kBM - 1) / kBM) * ((Nw + BN - 1) / BN);
            run += units * splits;
        }
        pre_s[E] = run;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_holder;
    const int total_units = pre_s[E];

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int issued = 0;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                const Unit t = decode_unit<BN, SWAP>(u, pre_s, cnt_s, E, Nw, splits, kb_total);
                const int tok_row = args.offsets[t.e] + t.tok0;
                for (int kb = t.kb0; kb < t.kb1; ++kb) {
                    if (!mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1u, status, tmo, 1)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = full0 + 8 * stage;
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    const int kx = kb * kBK;
                    if (!SWAP) {
                        tma_load_2d(sa, &tm_tok, fb, kx, tok_row);
                        tma_load_3d(sa + A_BYTES, &tm_w, fb, kx, t.w0, t.e);
                    } else {
                        tma_load_3d(sa, &tm_w, fb, kx, t.w0, t.e);
                        tma_load_2d(sa + A_BYTES, &tm_tok, fb, kx, tok_row);
                    }
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // let copies already in flight land before the CTA can exit
                int st = stage;
                uint32_t ph = phase;
                for (int i = 0; i < STAGES && i < issued; ++i) {
                    if (st == 0) {
                        st = STAGES - 1;
                        ph ^= 1u;
                    } else {
                        --st;
                    }
                    wait_drain(full0 + 8 * st, ph, tmo);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, any = false;
            int local = 0;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                const Unit t = decode_unit<BN, SWAP>(u, pre_s, cnt_s, E, Nw, splits, kb_total);
                const int acc = local & 1;
                const uint32_t acc_phase = (local >> 1) & 1;
                if (!mbar_wait_bounded(tempty0 + 8 * acc, acc_phase ^ 1u, status, tmo, 2)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                const int n_mma = (t.n_valid + 15) & ~15;
                const uint32_t idesc = idesc_bf16_f32(kBM, n_mma);
                for (int kb = t.kb0; kb < t.kb1; ++kb) {
                    if (!mbar_wait_bounded(full0 + 8 * stage, phase, status, tmo, 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const uint64_t ad = smem_desc_sw128(sa);
                    const uint64_t bd = smem_desc_sw128(sa + A_BYTES);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        // +32 bytes along K inside the 128-byte swizzled row = +2 in the
                        // descriptor's (address >> 4) field
                        umma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc,
                                  (kb > t.kb0 || kk > 0) ? 1u : 0u);
                    }
                    any = true;
                    umma_commit(empty0 + 8 * stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(tfull0 + 8 * acc);
                ++local;
            }
            if (!ok && any) {
                umma_commit(drain);
                wait_drain(drain, 0, tmo);
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;
        const int row_in_tile = q * 32 + lane;
        int local = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
            const Unit t = decode_unit<BN, SWAP>(u, pre_s, cnt_s, E, Nw, splits, kb_total);
            const int acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            if (!mbar_wait_warp(tfull0 + 8 * acc, acc_phase, status, tmo, 4)) break;
            tc_fence_after();
            const int cnt = cnt_s[t.e];
            const int64_t row_base = args.offsets[t.e];
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(acc * BN);
            const int chunks = (t.n_valid + 31) >> 5;
            for (int c = 0; c < chunks; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(taddr + c * 32, r);
                tmem_wait_ld();
                bias_act<EPI, SWAP>(r, args, t.e, t.w0 + c * 32, t.w0 + row_in_tile);
                if (!SWAP) {
                    const bool rv = t.tok0 + row_in_tile < cnt;
                    const int64_t grow = row_base + t.tok0 + row_in_tile;
                    const int col0 = t.w0 + c * 32;
                    if (EPI == EPI_F32) {
                        float *o = static_cast<float *>(args.out) + t.split * args.split_stride +
                                   grow * args.ldo;
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
                            const int col = col0 + 4 * g;
                            if (rv && col < Nw)
                                *reinterpret_cast<float4 *>(o + col) =
                                    make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                                                __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
                        }
                    } else {
                        __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(args.out) + grow * args.ldo;
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const int col = col0 + 8 * g;
                            if (rv && col < Nw) {
                                uint4 v;
                                __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    h[i] = __floats2bfloat162_rn(__uint_as_float(r[8 * g + 2 * i]),
                                                                 __uint_as_float(r[8 * g + 2 * i + 1]));
                                *reinterpret_cast<uint4 *>(o + col) = v;
                            }
                        }
                    }
                } else {
                    const int w = t.w0 + row_in_tile;
                    if (w < Nw) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int tok = t.tok0 + c * 32 + i;
                            if (tok < cnt) {
                                const int64_t grow = row_base + tok;
                                if (EPI == EPI_F32) {
                                    static_cast<float *>(args.out)[t.split * args.split_stride +
                                                                   grow * args.ldo + w] =
                                        __uint_as_float(r[i]);
                                } else {
                                    static_cast<__nv_bfloat16 *>(args.out)[grow * args.ldo + w] =
                                        __float2bfloat16_rn(__uint_as_float(r[i]));
                                }
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
            ++local;
        }
    }
    __syncwarp();
    __syncthreads();
    if (threadIdx.x == 0) publish_status(args.status, cta_status);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- CTA-pair variant (prefill)
// Two CTAs of a cluster share one 256 x 256 output tile (tcgen05 cta_group::2).
// Each CTA loads, per 64-wide K block, its own 128 token rows of A and its own
// 128 weight rows of B (plain TMA loads, no multicast) into a 6-stage ring; the
// bytes of both CTAs complete on the leader's (rank 0) barrier.  The leader's
// MMA lane issues M = 256, N = 256 MMAs that read A from each CTA's own shared
// memory and B from both, accumulating each CTA's 128 rows in that CTA's tensor
// memory; its commits arrive on both CTAs' barriers.  Both CTAs' epilogue warps
// drain their own accumulators and report to the leader's barrier.  Per byte
// moved from L2 this does a third more MMA work than the one-CTA tile, and each
// stage is 32 KB, so the ring is 50 % deeper.
//
// B_MN: the weights are stored [E][K][Nw] (K rows, Nw contiguous), as the
// backward reads W_down and W_up; each CTA then loads its 128 weight columns
// as two 64-wide MN-major boxes and the MMA reads B MN-major.
template <int EPI, int STAGES, bool B_MN = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
tc2_gemm_kernel(const __grid_constant__ CUtensorMap tm_tok, const __grid_constant__ CUtensorMap tm_w,
                const TcArgs args) {
    constexpr int BT = 256;                        // pair tile: 256 token rows x 256 weight rows
    constexpr uint32_t A_BYTES = 128 * kBK * 2;    // this CTA's 128 token rows
    constexpr uint32_t B_BYTES = 128 * kBK * 2;    // this CTA's 128 weight rows
    constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    constexpr uint32_t TMEM_COLS = 512;            // two 256-column accumulators

    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t bars[2 * STAGES + 5];
    __shared__ uint32_t tmem_holder;
    __shared__ int32_t pre_s[257];
    __shared__ int32_t cnt_s[256];
    __shared__ uint32_t cta_status;  // this CTA's copy of the status word

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int E = args.E, Nw = args.Nw, splits = args.splits;
    const int kb_total = (args.K + kBK - 1) / kBK;
    uint32_t *status = &cta_status;
    const uint64_t tmo = args.timeout_ns;

    const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    const uint32_t full0 = smem_u32(&bars[0]);
    const uint32_t empty0 = smem_u32(&bars[STAGES]);
    const uint32_t tfull0 = smem_u32(&bars[2 * STAGES]);
    const uint32_t tempty0 = smem_u32(&bars[2 * STAGES + 2]);
    const uint32_t drain = smem_u32(&bars[2 * STAGES + 4]);
    const uint32_t full0_lead = map_to_cta(full0, 0);
    const uint32_t tempty0_lead = map_to_cta(tempty0, 0);

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(tfull0, 1);
        mbar_init(tfull0 + 8, 1);
        mbar_init(tempty0, 8);       // 4 epilogue warps in each CTA
        mbar_init(tempty0 + 8, 8);
        mbar_init(drain, 1);
        fence_barrier_init();
        cta_status = 0u;
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_tok);
        tma_prefetch_desc(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&tmem_holder), TMEM_COLS);
        tmem_relinquish_pair();
    }
    pdl_wait();
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt_s[e] = args.counts[e];
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            pre_s[e] = run;
            run += ((cnt_s[e] + BT - 1) / BT) * ((Nw + BT - 1) / BT) * splits;
        }
        pre_s[E] = run;
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before either signals the other
    tc_fence_after();
    const uint32_t tmem_base = tmem_holder;
    const int total_units = pre_s[E];

    auto decode = [&](int u, int &e, int &tok0, int &w0, int &kb0, int &kb1, int &n_valid) {
        int lo = 0, hi = E;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre_s[mid] <= u) lo = mid; else hi = mid;
        }
        e = lo;
        int r = u - pre_s[lo];
        const int split = r % splits;
        r /= splits;
        // M tiles fastest: a wave of units shares the expert's token rows and a
        // few weight tiles (grouped M tiles and L2 eviction hints measured
        // slower on the Mixtral shape)
        const int mt = (cnt_s[lo] + BT - 1) / BT;
        tok0 = (r % mt) * BT;
        w0 = (r / mt) * BT;
        n_valid = min(BT, Nw - w0);
        kb0 = static_cast<int>(static_cast<int64_t>(split) * kb_total / splits);
        kb1 = static_cast<int>(static_cast<int64_t>(split + 1) * kb_total / splits);
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int issued = 0;
            const uint64_t pol = policy_evict_normal();
            for (int u = pair; u < total_units && ok; u += npairs) {
                int e, tok0, w0, kb0, kb1, nv;
                decode(u, e, tok0, w0, kb0, kb1, nv);
                const int tok_row = args.offsets[e] + tok0 + static_cast<int>(rank) * 128;
                const int w_row = w0 + static_cast<int>(rank) * 128;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1u, status, tmo, 11)) {
                        ok = false;
                        break;
                    }
                    if (leader) mbar_arrive_expect_tx(full0 + 8 * stage, 2 * STAGE_BYTES);
                    const uint32_t fb = full0_lead + 8 * stage;
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const int kx = kb * kBK;
                    tma_load_2d_pair(sa, &tm_tok, fb, kx, tok_row, pol);
                    if constexpr (B_MN) {
                        tma_load_3d_pair(sa + A_BYTES, &tm_w, fb, w_row, kx, e, pol);
                        tma_load_3d_pair(sa + A_BYTES + 8192u, &tm_w, fb, w_row + 64, kx, e, pol);
                    } else {
                        tma_load_3d_pair(sa + A_BYTES, &tm_w, fb, kx, w_row, e, pol);
                    }
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && leader) {
                // the pair's copies of the stages armed here land before exit
                int st = stage;
                uint32_t ph = phase;
                for (int i = 0; i < STAGES && i < issued; ++i) {
                    if (st == 0) {
                        st = STAGES - 1;
                        ph ^= 1u;
                    } else {
                        --st;
                    }
                    wait_drain(full0 + 8 * st, ph, tmo);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, any = false;
            int local = 0;
            const uint32_t idesc = idesc_bf16_f32(256, 256) | (B_MN ? kIdescBMajorMN : 0u);
            for (int u = pair; u < total_units && ok; u += npairs) {
                int e, tok0, w0, kb0, kb1, nv;
                decode(u, e, tok0, w0, kb0, kb1, nv);
                const int acc = local & 1;
                const uint32_t acc_phase = (local >> 1) & 1;
                if (!mbar_wait_bounded(tempty0 + 8 * acc, acc_phase ^ 1u, status, tmo, 12)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BT);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(full0 + 8 * stage, phase, status, tmo, 13)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const uint64_t ad = smem_desc_sw128(sa);
                    // MN-major B: 64-wide N blocks 8 KB apart, 8-row K groups 1 KB
                    // apart; the next 16 K rows start 2 KB on (+128 in the field)
                    const uint64_t bd = B_MN ? smem_desc_mn_sw128(sa + A_BYTES, 8192u, 1024u)
                                             : smem_desc_sw128(sa + A_BYTES);
                    constexpr uint32_t bstep = B_MN ? 128u : 2u;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_bf16_pair(d_tmem, ad + 2 * kk, bd + bstep * kk, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
                    any = true;
                    umma_commit_pair_mc(empty0 + 8 * stage, 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair_mc(tfull0 + 8 * acc, 0x3);
                ++local;
            }
            if (!ok && any) {
                umma_commit_pair(drain);
                wait_drain(drain, 0, tmo);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int row_in_tile = q * 32 + lane;
        int local = 0;
        for (int u = pair; u < total_units; u += npairs) {
            int e, tok0, w0, kb0, kb1, nv;
            decode(u, e, tok0, w0, kb0, kb1, nv);
            const int acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            if (!mbar_wait_warp(tfull0 + 8 * acc, acc_phase, status, tmo, 14)) break;
            tc_fence_after();
            const int cnt = cnt_s[e];
            const int my_row = tok0 + static_cast<int>(rank) * 128 + row_in_tile;
            const bool rv = my_row < cnt;
            const int64_t grow = static_cast<int64_t>(args.offsets[e]) + my_row;
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(acc * BT);
            const int chunks = (nv + 31) >> 5;
            for (int c = 0; c < chunks; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(taddr + c * 32, r);
                tmem_wait_ld();
                bias_act<EPI, false>(r, args, e, w0 + c * 32, 0);
                const int col0 = w0 + c * 32;
                if constexpr (EPI == EPI_BF16_MASK) {
                    if (rv) {
                        const __nv_bfloat16 *mk = args.mask + grow * args.ldo + col0;
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            if (col0 + 8 * g < Nw) {
                                uint4 mv = *reinterpret_cast<const uint4 *>(mk + 8 * g);
                                const __nv_bfloat16 *mb = reinterpret_cast<const __nv_bfloat16 *>(&mv);
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    if (!(__bfloat162float(mb[i]) > 0.0f)) r[8 * g + i] = 0u;
                            }
                        }
                    }
                }
                __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(args.out) + grow * args.ldo;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int col = col0 + 8 * g;
                    if (rv && col < Nw) {
                        uint4 v;
                        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            h[i] = __floats2bfloat162_rn(__uint_as_float(r[8 * g + 2 * i]),
                                                         __uint_as_float(r[8 * g + 2 * i + 1]));
                        *reinterpret_cast<uint4 *>(o + col) = v;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(tempty0 + 8 * acc);
                else mbar_arrive_cluster(tempty0_lead + 8 * acc);
            }
            ++local;
        }
    }
    __syncwarp();
    __syncthreads();
    if (threadIdx.x == 0) publish_status(args.status, cta_status);
    cluster_sync();  // the pair's MMAs and remote arrivals are done before TMEM goes
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

template <int BN, bool SWAP, int EPI, int STAGES>
cudaError_t launch_tc(const void *tok, int64_t tok_rows, const void *W, int E, int Nw, int K,
                      const int32_t *offsets, const int32_t *counts, int splits, void *out,
                      int64_t ldo, int64_t split_stride, uint32_t *status, uint64_t timeout_ns,
                      int grid, cudaStream_t s, const float *bias = nullptr, int act = 1) {
    CUtensorMap tm_tok, tm_w;
    if (!make_tmap_bf16_2d(&tm_tok, tok, tok_rows, K, SWAP ? BN : kBM)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_3d(&tm_w, W, E, Nw, K, SWAP ? kBM : BN)) return cudaErrorInvalidValue;
    constexpr int smem = STAGES * (kBM + BN) * kBK * 2 + 1024;
    auto kern = tc_gemm_kernel<BN, SWAP, EPI, STAGES>;
    // every call: the attribute belongs to the current device's context
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    TcArgs a{offsets, counts, E, Nw, K, splits, out, ldo, split_stride, status, timeout_ns, bias, act, nullptr};
    return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, s, tm_tok, tm_w, a);
}

template <int EPI, int STAGES, bool B_MN = false>
cudaError_t launch_tc2(const void *tok, int64_t tok_rows, const void *W, int E, int Nw, int K,
                       const int32_t *offsets, const int32_t *counts, void *out, int64_t ldo,
                       uint32_t *status, uint64_t timeout_ns, int num_sms, cudaStream_t s,
                       const float *bias = nullptr, int act = 1, const void *mask = nullptr) {
    CUtensorMap tm_tok, tm_w;
    if (!make_tmap_bf16_2d(&tm_tok, tok, tok_rows, K, 128)) return cudaErrorInvalidValue;
    if (B_MN) {
        // W is [E][K][Nw]: boxes of 64 weight columns x 64 K rows
        if (!make_tmap_bf16_3d(&tm_w, W, E, K, Nw, 64)) return cudaErrorInvalidValue;
    } else {
        if (!make_tmap_bf16_3d(&tm_w, W, E, Nw, K, 128)) return cudaErrorInvalidValue;
    }
    constexpr int smem = STAGES * 2 * 128 * kBK * 2 + 1024;
    auto kern = tc2_gemm_kernel<EPI, STAGES, B_MN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int pairs = num_sms / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    int max_clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) == cudaSuccess && max_clusters > 0 &&
        max_clusters < pairs)
        pairs = max_clusters;
    (void)cudaGetLastError();
    TcArgs a{offsets, counts, E, Nw, K, 1, out, ldo, 0, status, timeout_ns, bias, act,
             static_cast<const __nv_bfloat16 *>(mask)};
    return launch_pdl(kern, dim3(2 * pairs), dim3(kThreads), smem, s, tm_tok, tm_w, a);
}

// ---------------------------------------------------------------- weight gradients
// D[e][m][n] = sum over expert e's gathered rows r of P[r][m] * Q[r][n], fp32
// out: the backward's dW_down[e] = dO^T H and dW_up[e] = dZ^T X.  The GEMM's
// K is the expert's rows, so both operands are read MN-major: per 64-row K
// block the CTA loads its 128 columns of P (two 64-wide boxes, A) and 256
// columns of Q (four boxes, B).  The rows of a K block past the expert's last
// row belong to the next expert (the layout has no padding): before the MMAs
// of that block the MMA warp overwrites those K rows with zeros in shared
// memory.  An expert without rows gets a zero tile without MMAs.
// Warp roles as in tc_gemm_kernel; units (expert, M tile, N tile), with the
// operand whose tile set is smaller walked fastest so it stays in L2.
struct WgArgs {
    const int32_t *offsets;
    const int32_t *counts;
    int E, M, Nn;  // D[e] is [M][Nn]
    int m_fast;    // 1: M tiles fastest
    float *out;
    uint32_t *status;
    uint64_t timeout_ns;
};

constexpr int kWM = 128, kWN = 256;

template <int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
tc_wgrad_kernel(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_q,
                const WgArgs args) {
    constexpr uint32_t A_BYTES = kWM * kBK * 2;   // two 8 KB boxes
    constexpr uint32_t B_BYTES = kWN * kBK * 2;   // four 8 KB boxes
    constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    constexpr uint32_t TMEM_COLS = 2 * kWN;
    static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");

    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t bars[2 * STAGES + 5];
    __shared__ uint32_t tmem_holder;
    __shared__ int32_t cnt_s[256];
    __shared__ int32_t off_s[256];
    __shared__ uint32_t cta_status;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = args.E, M = args.M, Nn = args.Nn;
    const int mt = (M + kWM - 1) / kWM, nt = (Nn + kWN - 1) / kWN;
    const int total_units = E * mt * nt;
    uint32_t *status = &cta_status;
    const uint64_t tmo = args.timeout_ns;

    const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    uint8_t *smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
    const uint32_t full0 = smem_u32(&bars[0]);
    const uint32_t empty0 = smem_u32(&bars[STAGES]);
    const uint32_t tfull0 = smem_u32(&bars[2 * STAGES]);
    const uint32_t tempty0 = smem_u32(&bars[2 * STAGES + 2]);
    const uint32_t drain = smem_u32(&bars[2 * STAGES + 4]);

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(tfull0, 1);
        mbar_init(tfull0 + 8, 1);
        mbar_init(tempty0, 4);
        mbar_init(tempty0 + 8, 4);
        mbar_init(drain, 1);
        fence_barrier_init();
        cta_status = 0u;
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_p);
        tma_prefetch_desc(&tm_q);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tmem_holder), TMEM_COLS);
        tmem_relinquish();
    }
    pdl_wait();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        cnt_s[e] = args.counts[e];
        off_s[e] = args.offsets[e];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_holder;

    auto decode = [&](int u, int &e, int &m, int &n) {
        e = u / (mt * nt);
        const int r = u - e * (mt * nt);
        if (args.m_fast) {
            m = r % mt;
            n = r / mt;
        } else {
            m = r / nt;
            n = r % nt;
        }
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                int e, m, n;
                decode(u, e, m, n);
                const int nk = (cnt_s[e] + kBK - 1) / kBK;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1u, status, tmo, 31)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = full0 + 8 * stage;
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    const int y = off_s[e] + kb * kBK;
#pragma unroll
                    for (int h = 0; h < 2; ++h) tma_load_2d(sa + h * 8192u, &tm_p, fb, m * kWM + h * 64, y);
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        tma_load_2d(sa + A_BYTES + h * 8192u, &tm_q, fb, n * kWN + h * 64, y);
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                int st = stage;
                uint32_t ph = phase;
                for (int i = 0; i < STAGES && i < issued; ++i) {
                    if (st == 0) {
                        st = STAGES - 1;
                        ph ^= 1u;
                    } else {
                        --st;
                    }
                    wait_drain(full0 + 8 * st, ph, tmo);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ tail zeroing + MMA issue (whole warp)
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true, any = false;
        int local = 0;
        const uint32_t idesc = idesc_bf16_f32(kWM, kWN) | kIdescAMajorMN | kIdescBMajorMN;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
            int e, m, n;
            decode(u, e, m, n);
            const int cnt = cnt_s[e];
            const int nk = (cnt + kBK - 1) / kBK;
            if (nk == 0) continue;
            const int acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            if (!mbar_wait_warp(tempty0 + 8 * acc, acc_phase ^ 1u, status, tmo, 32)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kWN);
            for (int kb = 0; kb < nk; ++kb) {
                if (!mbar_wait_warp(full0 + 8 * stage, phase, status, tmo, 33)) {
                    ok = false;
                    break;
                }
                const int v = cnt - kb * kBK;  // valid K rows of this block
                if (v < kBK) {
                    uint8_t *st = smem_gen + stage * STAGE_BYTES;
                    const int per_box = (kBK - v) * 8;  // 16-byte chunks past the last row
                    for (int q = lane; q < 6 * per_box; q += 32) {
                        const int box = q / per_box, rem = q - box * per_box;
                        *reinterpret_cast<uint4 *>(st + box * 8192 + (v + rem / 8) * 128 + (rem % 8) * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();  // the zeros, visible to the MMA
                }
                __syncwarp();
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const uint64_t ad = smem_desc_mn_sw128(sa, 8192u, 1024u);
                    const uint64_t bd = smem_desc_mn_sw128(sa + A_BYTES, 8192u, 1024u);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_bf16(d_tmem, ad + 128u * kk, bd + 128u * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(empty0 + 8 * stage);
                }
                any = true;
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(tfull0 + 8 * acc);
            ++local;
        }
        if (!ok && any && lane == 0) {
            umma_commit(drain);
            wait_drain(drain, 0, tmo);
        }
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;
        const int row_in_tile = q * 32 + lane;
        int local = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
            int e, m, n;
            decode(u, e, m, n);
            const int mrow = m * kWM + row_in_tile;
            float *o = args.out + (static_cast<int64_t>(e) * M + mrow) * Nn;
            if (cnt_s[e] == 0) {
                // no rows: a zero gradient, without touching the tensor memory
                if (mrow < M)
                    for (int c = n * kWN; c < n * kWN + kWN && c < Nn; c += 4)
                        *reinterpret_cast<float4 *>(o + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                continue;
            }
            const int acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            if (!mbar_wait_warp(tfull0 + 8 * acc, acc_phase, status, tmo, 34)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(acc * kWN);
            for (int c = 0; c < kWN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(taddr + c * 32, r);
                tmem_wait_ld();
                const int col0 = n * kWN + c * 32;
                if (mrow < M) {
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const int col = col0 + 4 * g;
                        if (col < Nn)
                            *reinterpret_cast<float4 *>(o + col) =
                                make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                                            __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
            ++local;
        }
    }
    __syncwarp();
    __syncthreads();
    if (threadIdx.x == 0) publish_status(args.status, cta_status);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// The weight gradients on CTA pairs (tcgen05 cta_group::2): a pair computes a
// 256 x 256 tile of D[e], CTA r holding the M columns [r 128, r 128 + 128) of
// the tile's P block (A) and the N columns [r 128, r 128 + 128) of its Q block
// (B); the leader's MMA reads B from both CTAs and each CTA accumulates its 128
// rows of D in its own tensor memory.  Per K block a CTA moves 32 KB through
// TMA, where the one-CTA tile moves 48 KB for half the MMA work.
// Both CTAs' loads complete on the leader's barrier (as in tc2_gemm_kernel).
// The K rows past the expert's last row, in the last K block of a unit, are
// zeroed by the leader's MMA warp in both CTAs' shared memory (the peer's
// through the cluster window), behind a cluster-scope proxy fence, before it
// issues that block's MMAs.
template <int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
tc_wgrad2_kernel(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_q,
                 const WgArgs args) {
    constexpr int BT = 256;                        // pair tile: 256 M x 256 N
    constexpr uint32_t A_BYTES = 128 * kBK * 2;    // this CTA's 128 M columns: two 8 KB boxes
    constexpr uint32_t B_BYTES = 128 * kBK * 2;    // this CTA's 128 N columns: two 8 KB boxes
    constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    constexpr uint32_t TMEM_COLS = 512;            // two 256-column accumulators
    static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");

    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t bars[2 * STAGES + 5];
    __shared__ uint32_t tmem_holder;
    __shared__ int32_t cnt_s[256];
    __shared__ int32_t off_s[256];
    __shared__ uint32_t cta_status;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int E = args.E, M = args.M, Nn = args.Nn;
    const int mt = (M + BT - 1) / BT, nt = (Nn + BT - 1) / BT;
    const int total_units = E * mt * nt;
    uint32_t *status = &cta_status;
    const uint64_t tmo = args.timeout_ns;

    const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    uint8_t *smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
    const uint32_t full0 = smem_u32(&bars[0]);                // [STAGES] both CTAs' loads (leader's counts)
    const uint32_t empty0 = smem_u32(&bars[STAGES]);          // [STAGES] the pair's MMAs are done
    const uint32_t tfull0 = smem_u32(&bars[2 * STAGES]);
    const uint32_t tempty0 = smem_u32(&bars[2 * STAGES + 2]);
    const uint32_t drain = smem_u32(&bars[2 * STAGES + 4]);
    const uint32_t full0_lead = map_to_cta(full0, 0);
    const uint32_t tempty0_lead = map_to_cta(tempty0, 0);

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(tfull0, 1);
        mbar_init(tfull0 + 8, 1);
        mbar_init(tempty0, 8);  // 4 epilogue warps in each CTA
        mbar_init(tempty0 + 8, 8);
        mbar_init(drain, 1);
        fence_barrier_init();
        cta_status = 0u;
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_p);
        tma_prefetch_desc(&tm_q);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&tmem_holder), TMEM_COLS);
        tmem_relinquish_pair();
    }
    pdl_wait();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        cnt_s[e] = args.counts[e];
        off_s[e] = args.offsets[e];
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before either signals the other
    tc_fence_after();
    const uint32_t tmem_base = tmem_holder;

    auto decode = [&](int u, int &e, int &m, int &n) {
        e = u / (mt * nt);
        const int r = u - e * (mt * nt);
        if (args.m_fast) {
            m = r % mt;
            n = r / mt;
        } else {
            m = r / nt;
            n = r % nt;
        }
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            const uint64_t pol = policy_evict_normal();
            for (int u = pair; u < total_units && ok; u += npairs) {
                int e, m, n;
                decode(u, e, m, n);
                const int nk = (cnt_s[e] + kBK - 1) / kBK;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1u, status, tmo, 41)) {
                        ok = false;
                        break;
                    }
                    if (leader) mbar_arrive_expect_tx(full0 + 8 * stage, 2 * STAGE_BYTES);
                    const uint32_t fb = full0_lead + 8 * stage;
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const int y = off_s[e] + kb * kBK;
                    const int mc = m * BT + static_cast<int>(rank) * 128, nc = n * BT + static_cast<int>(rank) * 128;
#pragma unroll
                    for (int h = 0; h < 2; ++h) tma_load_2d_pair(sa + h * 8192u, &tm_p, fb, mc + h * 64, y, pol);
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d_pair(sa + A_BYTES + h * 8192u, &tm_q, fb, nc + h * 64, y, pol);
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && leader) {
                // the pair's copies of the stages armed here land before exit
                int st = stage;
                uint32_t ph = phase;
                for (int i = 0; i < STAGES && i < issued; ++i) {
                    if (st == 0) {
                        st = STAGES - 1;
                        ph ^= 1u;
                    } else {
                        --st;
                    }
                    wait_drain(full0 + 8 * st, ph, tmo);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ tail zeroing + MMA issue (leader, whole warp)
        if (leader) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, any = false;
            int local = 0;
            const uint32_t idesc = idesc_bf16_f32(BT, BT) | kIdescAMajorMN | kIdescBMajorMN;
            for (int u = pair; u < total_units && ok; u += npairs) {
                int e, m, n;
                decode(u, e, m, n);
                const int cnt = cnt_s[e];
                const int nk = (cnt + kBK - 1) / kBK;
                if (nk == 0) continue;
                const int acc = local & 1;
                const uint32_t acc_phase = (local >> 1) & 1;
                if (!mbar_wait_warp(tempty0 + 8 * acc, acc_phase ^ 1u, status, tmo, 42)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BT);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait_warp(full0 + 8 * stage, phase, status, tmo, 43)) {
                        ok = false;
                        break;
                    }
                    const int v = cnt - kb * kBK;  // valid K rows of this block
                    if (v < kBK) {
                        // rows v.. of the four boxes, in this CTA and in the peer
                        const uint32_t st = smem_base + stage * STAGE_BYTES;
                        const uint32_t st_peer = map_to_cta(st, 1);
                        const int per_box = (kBK - v) * 8;  // 16-byte chunks past the last row
                        for (int q = lane; q < 4 * per_box; q += 32) {
                            const int box = q / per_box, rem = q - box * per_box;
                            const uint32_t off = static_cast<uint32_t>(box * 8192 + (v + rem / 8) * 128 + (rem % 8) * 16);
                            *reinterpret_cast<uint4 *>(smem_gen + stage * STAGE_BYTES + off) = make_uint4(0u, 0u, 0u, 0u);
                            st_shared_cluster_zero16(st_peer + off);
                        }
                        fence_proxy_async_smem();
                        fence_proxy_async_cluster();  // the zeros, visible to the MMA in both CTAs
                    }
                    __syncwarp();
                    if (lane == 0) {
                        tc_fence_after();
                        const uint32_t sa = smem_base + stage * STAGE_BYTES;
                        const uint64_t ad = smem_desc_mn_sw128(sa, 8192u, 1024u);
                        const uint64_t bd = smem_desc_mn_sw128(sa + A_BYTES, 8192u, 1024u);
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk)
                            umma_bf16_pair(d_tmem, ad + 128u * kk, bd + 128u * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                        umma_commit_pair_mc(empty0 + 8 * stage, 0x3);
                    }
                    any = true;
                    __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) umma_commit_pair_mc(tfull0 + 8 * acc, 0x3);
                ++local;
            }
            if (!ok && any && lane == 0) {
                umma_commit_pair(drain);
                wait_drain(drain, 0, tmo);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int row_in_tile = q * 32 + lane;
        int local = 0;
        for (int u = pair; u < total_units; u += npairs) {
            int e, m, n;
            decode(u, e, m, n);
            const int mrow = m * BT + static_cast<int>(rank) * 128 + row_in_tile;
            float *o = args.out + (static_cast<int64_t>(e) * M + mrow) * Nn;
            if (cnt_s[e] == 0) {
                // no rows: a zero gradient, without touching the tensor memory
                if (mrow < M)
                    for (int c = n * BT; c < n * BT + BT && c < Nn; c += 4)
                        *reinterpret_cast<float4 *>(o + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                continue;
            }
            const int acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            if (!mbar_wait_warp(tfull0 + 8 * acc, acc_phase, status, tmo, 45)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BT);
            for (int c = 0; c < BT / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(taddr + c * 32, r);
                tmem_wait_ld();
                const int col0 = n * BT + c * 32;
                if (mrow < M) {
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const int col = col0 + 4 * g;
                        if (col < Nn)
                            *reinterpret_cast<float4 *>(o + col) =
                                make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]),
                                            __uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(tempty0 + 8 * acc);
                else mbar_arrive_cluster(tempty0_lead + 8 * acc);
            }
            ++local;
        }
    }
    __syncwarp();
    __syncthreads();
    if (threadIdx.x == 0) publish_status(args.status, cta_status);
    cluster_sync();  // the pair's MMAs and remote arrivals are done before the tensor memory goes
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// MOE_WGRAD_PAIR=0 keeps the weight gradients on single CTAs (for comparisons).
bool wgrad_pair_enabled() {
    static const bool on = [] {
        const char *v = getenv("MOE_WGRAD_PAIR");
        return v == nullptr || atoi(v) != 0;
    }();
    return on;
}

cudaError_t launch_wgrad(const void *P, const void *Q, int64_t rows, int M, int Nn, const int32_t *offsets,
                         const int32_t *counts, int E, float *out, uint32_t *status, uint64_t timeout_ns,
                         int num_sms, cudaStream_t s) {
    constexpr int STAGES = 4;
    CUtensorMap tm_p, tm_q;
    if (!make_tmap_bf16_2d(&tm_p, P, rows, M, 64)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tm_q, Q, rows, Nn, 64)) return cudaErrorInvalidValue;
    constexpr int smem = STAGES * (kWM + kWN) * kBK * 2 + 1024;
    auto kern = tc_wgrad_kernel<STAGES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    WgArgs a{offsets, counts, E, M, Nn, M <= Nn ? 1 : 0, out, status, timeout_ns};
    if (num_sms >= 2 && wgrad_pair_enabled()) {
        // CTA pairs, 256 x 256 tiles
        constexpr int STAGES2 = 6;
        constexpr int smem2 = STAGES2 * 2 * 128 * kBK * 2 + 1024;
        auto kern2 = tc_wgrad2_kernel<STAGES2>;
        e = cudaFuncSetAttribute(kern2, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
        if (e != cudaSuccess) return e;
        const int units2 = E * ((M + 255) / 256) * ((Nn + 255) / 256);
        const int pairs = units2 < num_sms / 2 ? units2 : num_sms / 2;
        return launch_pdl(kern2, dim3(2 * (pairs > 0 ? pairs : 1)), dim3(kThreads), smem2, s, tm_p, tm_q, a);
    }
    const int units = E * ((M + kWM - 1) / kWM) * ((Nn + kWN - 1) / kWN);
    const int grid = units < num_sms ? units : num_sms;
    return launch_pdl(kern, dim3(grid > 0 ? grid : 1), dim3(kThreads), smem, s, tm_p, tm_q, a);
}

// Sum of K-split fp32 partials into bf16 rows, in split order, then the
// expert's bias (nullable, [E][d]) and the activation (0 none, 1 ReLU,
// 2 GELU).  Only the kept rows (below offsets[E]) are touched.
__global__ void __launch_bounds__(256)
reduce_parts_kernel(const float *__restrict__ parts, int nparts, int64_t part_stride,
                    const int32_t *__restrict__ offsets, int E, int d, const float *__restrict__ bias,
                    int act, __nv_bfloat16 *__restrict__ out) {
    pdl_trigger();
    pdl_wait();
    const int64_t rows = offsets[E];
    const int q = d / 4;
    const int64_t total = rows * q;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float4 a = reinterpret_cast<const float4 *>(parts)[i];
        for (int p = 1; p < nparts; ++p) {
            const float4 b = reinterpret_cast<const float4 *>(parts + p * part_stride)[i];
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        if (bias != nullptr) {
            const int64_t row = i / q;
            const int c = static_cast<int>(i - row * q) * 4;
            int lo = 0, hi = E;  // offsets[lo] <= row < offsets[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (offsets[mid] <= row) lo = mid; else hi = mid;
            }
            const float4 bb = *reinterpret_cast<const float4 *>(bias + static_cast<int64_t>(lo) * d + c);
            a.x += bb.x; a.y += bb.y; a.z += bb.z; a.w += bb.w;
        }
        if (act != 0) {
            a.x = activate(a.x, act); a.y = activate(a.y, act);
            a.z = activate(a.z, act); a.w = activate(a.w, act);
        }
        __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(out) + 2 * i;
        o[0] = __floats2bfloat162_rn(a.x, a.y);
        o[1] = __floats2bfloat162_rn(a.z, a.w);
    }
}

}  // namespace

// K splits that give about `waves` units per SM for `units` equal tiles.
int decode_splits(int64_t units, int K, int num_sms, int64_t waves) {
    const int kb_total = (K + kBK - 1) / kBK;
    int s = static_cast<int>((waves * num_sms + units - 1) / units);
    if (s > 8) s = 8;
    if (s > kb_total) s = kb_total;
    if (s < 1) s = 1;
    return s;
}

TcPlan plan_tc_ffn(int64_t rows, int d, int d_ff, int E, int num_sms) {
    TcPlan p{};
    p.decode = rows <= 256;
    p.splits_up = 1;
    p.splits_down = 1;
    // CTA-pair tiles for prefill; MOE_TC_PAIR=0 selects the one-CTA tiles
    static const int pair_env = [] {
        const char *v = getenv("MOE_TC_PAIR");
        return v ? atoi(v) : 1;
    }();
    p.pair = !p.decode && pair_env != 0 && num_sms >= 2;
    if (p.decode) {
        // weight-streaming tiles: enough equal units that the last wave is a
        // small part of the whole, split over K (fp32 partials) to get there
        // (the combine reads every down partial, so that one aims lower).  At
        // the Mixtral shape the up projection's 896 weight tiles give 18.2
        // waves with three splits, where two left 16 units in a 13th wave.
        p.splits_up = decode_splits(static_cast<int64_t>(E) * ((d_ff + kBM - 1) / kBM), d, num_sms, 18);
        p.splits_down = decode_splits(static_cast<int64_t>(E) * ((d + kBM - 1) / kBM), d_ff, num_sms, 6);
    }
    return p;
}

size_t tc_ffn_ws_bytes(int64_t rows, int d, int d_ff, int E, int num_sms) {
    const TcPlan p = plan_tc_ffn(rows, d, d_ff, E, num_sms);
    size_t b = align_up(static_cast<size_t>(rows) * d_ff * 2, 256);  // hidden activations
    if (p.decode) {
        b += align_up(static_cast<size_t>(p.splits_down) * rows * d * 4, 256);
        if (p.splits_up > 1) b += align_up(static_cast<size_t>(p.splits_up) * rows * d_ff * 4, 256);
    }
    return b;
}

int tc_ffn_launches(const TcPlan &p, bool combine_reads_parts) {
    if (!p.decode) return 2;
    return 2 + (p.splits_up > 1 ? 1 : 0) + (combine_reads_parts ? 0 : 1);
}

cudaError_t launch_tc_ffn(const void *xg, const int32_t *offsets, const int32_t *counts,
                          const void *W_up, const void *W_down, int64_t rows, int d, int d_ff,
                          int E, void *out, void *H, float *parts, bool combine_reads_parts,
                          uint32_t *status, uint64_t timeout_ns, int num_sms, cudaStream_t s,
                          TcPlan *plan_out, int act, const float *b_up, const float *b_down) {
    const TcPlan p = plan_tc_ffn(rows, d, d_ff, E, num_sms);
    if (plan_out) *plan_out = p;
    cudaError_t e;
    if (!p.decode && p.pair) {
        if (act == 1 && b_up == nullptr)
            e = launch_tc2<EPI_BF16_RELU, 6>(xg, rows, W_up, E, d_ff, d, offsets, counts, H, d_ff, status,
                                             timeout_ns, num_sms, s);
        else
            e = launch_tc2<EPI_BF16_ACT, 6>(xg, rows, W_up, E, d_ff, d, offsets, counts, H, d_ff, status,
                                            timeout_ns, num_sms, s, b_up, act);
        if (e != cudaSuccess) return e;
        if (b_down == nullptr)
            return launch_tc2<EPI_BF16_PLAIN, 6>(H, rows, W_down, E, d, d_ff, offsets, counts, out, d, status,
                                                 timeout_ns, num_sms, s);
        return launch_tc2<EPI_BF16, 6>(H, rows, W_down, E, d, d_ff, offsets, counts, out, d, status,
                                       timeout_ns, num_sms, s, b_down, 0);
    }
    if (!p.decode) {
        e = launch_tc<256, false, EPI_BF16_ACT, 4>(xg, rows, W_up, E, d_ff, d, offsets, counts, 1, H,
                                                   d_ff, 0, status, timeout_ns, num_sms, s, b_up, act);
        if (e != cudaSuccess) return e;
        return launch_tc<256, false, EPI_BF16, 4>(H, rows, W_down, E, d, d_ff, offsets, counts, 1, out,
                                                  d, 0, status, timeout_ns, num_sms, s, b_down, 0);
    }
    if (p.splits_up > 1) {
        // up projection split over K into fp32 partials, then ReLU of their sum
        float *parts_up = parts + align_up(static_cast<size_t>(p.splits_down) * rows * d * 4, 256) / 4;
        const int64_t ustride = rows * static_cast<int64_t>(d_ff);
        e = launch_tc<64, true, EPI_F32, 8>(xg, rows, W_up, E, d_ff, d, offsets, counts, p.splits_up, parts_up,
                                            d_ff, ustride, status, timeout_ns, num_sms, s);
        if (e != cudaSuccess) return e;
        const int64_t total_h = rows * (d_ff / 4);
        const int hblocks =
            static_cast<int>((total_h + 255) / 256 < 4 * num_sms ? (total_h + 255) / 256 : 4 * num_sms);
e = launch_pdl(reduce_parts_kernel, dim3(hblocks > 0 ? hblocks : 1), dim3(256), 0, s,
                       static_cast<const float *>(parts_up), p.splits_up, ustride,
                       static_cast<const int32_t *>(offsets), E, d_ff, b_up, act, static_cast<__nv_bfloat16 *>(H));
    } else {
        e = launch_tc<64, true, EPI_BF16_ACT, 8>(xg, rows, W_up, E, d_ff, d, offsets, counts, 1, H, d_ff, 0,
                                                 status, timeout_ns, num_sms, s, b_up, act);
    }
    if (e != cudaSuccess) return e;
    const int64_t pstride = rows * static_cast<int64_t>(d);
    e = launch_tc<64, true, EPI_F32, 8>(H, rows, W_down, E, d, d_ff, offsets, counts, p.splits_down,
                                        parts, d, pstride, status, timeout_ns, num_sms, s);
    if (e != cudaSuccess || combine_reads_parts) return e;
    const int64_t total = rows * (d / 4);
    const int blocks = static_cast<int>((total + 255) / 256 < 4 * num_sms ? (total + 255) / 256 : 4 * num_sms);
    return launch_pdl(reduce_parts_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, s,
                      static_cast<const float *>(parts), p.splits_down, pstride, static_cast<const int32_t *>(offsets),
                      E, d, b_down, 0, static_cast<__nv_bfloat16 *>(out));
}

cudaError_t launch_tc_bwd_gemms(const BwdArgs &a, const void *dO, void *dZ, void *dX, uint32_t *status,
                                uint64_t timeout_ns, int num_sms, cudaStream_t s) {
    // dZ = (dO W_down[e]) * [H > 0]: tokens dO [rows][d] (K = d), W_down [E][d][d_ff] read MN-major
    cudaError_t e = launch_tc2<EPI_BF16_MASK, 6, true>(dO, a.rows, a.W_down, a.E, a.d_ff, a.d, a.offsets, a.counts,
                                                       dZ, a.d_ff, status, timeout_ns, num_sms, s, nullptr, 1, a.H);
    if (e != cudaSuccess) return e;
    // dX = dZ W_up[e]: tokens dZ [rows][d_ff] (K = d_ff), W_up [E][d_ff][d] read MN-major
    e = launch_tc2<EPI_BF16_PLAIN, 6, true>(dZ, a.rows, a.W_up, a.E, a.d, a.d_ff, a.offsets, a.counts, dX, a.d, status,
                                      timeout_ns, num_sms, s);
    if (e != cudaSuccess) return e;
    // dW_down[e] = dO^T H ([d][d_ff]), dW_up[e] = dZ^T X ([d_ff][d])
    e = launch_wgrad(dO, a.H, a.rows, a.d, a.d_ff, a.offsets, a.counts, a.E, a.dW_down, status, timeout_ns, num_sms,
                     s);
    if (e != cudaSuccess) return e;
    return launch_wgrad(dZ, a.x_gathered, a.rows, a.d_ff, a.d, a.offsets, a.counts, a.E, a.dW_up, status,
                        timeout_ns, num_sms, s);
}

// Diagnostic: one CTA waits on a barrier that nothing completes.
__global__ void wait_timeout_kernel(uint32_t *status, uint64_t timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t cta_status;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
        cta_status = 0u;
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(b, 0, &cta_status, timeout_ns, 9);
    __syncthreads();
    if (threadIdx.x == 0) publish_status(status, cta_status);
}

cudaError_t launch_wait_timeout(uint32_t *status, uint64_t timeout_ns, cudaStream_t s) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace moe
