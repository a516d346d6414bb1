// Router on the fifth-generation tensor cores, for bf16 tokens: logits, noise,
// KeepTopK and softmax over the kept scores in one kernel.
//
// "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 2 (s_raw = W_g x),
// STEP 4 (s = s_raw + eps), STEP 5 (-inf outside the top k), STEP 6 (softmax);
// "nanoMoEの深層解剖" slides 11-13 (the router runs in fp32 with autocast
// disabled: logits, topk, -inf scatter, softmax).
//
// fp32 products on bf16 tensor cores.  Each fp32 router weight is cut into
// three bf16 parts, w = w_hi + w_mid + w_lo, each part the round-to-nearest
// bf16 of what the parts before it left over.  The remainders are exact in
// fp32 and the three 8-bit significands hold all 24 bits of w, so the sum is
// w itself.  A bf16 token value times a bf16 part is exact in fp32 (16
// significant bits), so every product the MMA forms is the exact fp32 product
// x*w split in three; only the accumulation rounds, in fp32, as a CUDA-core
// dot product would.  The three part-sums are added in the order hi, mid, lo.
//
// Tile: 128 tokens (MMA M) x all experts.  B is the 3*E_pad rows
// [w_hi of experts 0..E_pad-1; w_mid ...; w_lo ...] of one 64-wide K block,
// written by the CTA's own threads into the 128-byte-swizzled K-major layout
// the MMA reads; x arrives by TMA.  Accumulators: 3*E_pad fp32 columns of
// tensor memory (column c = row c of B).
//
// Warp roles (192 threads): warp 0 lane 0 issues the x TMA loads into a
// STAGES-deep ring; warp 1 owns the tensor memory and its lane 0 issues the
// MMAs; warps 2-5 split W_g into the ring's B slots, then run the epilogue
// (warp w reads TMEM lanes 32*(w%4)..+31, one token per thread): add the
// three parts and the bias, write the logits (coalesced, through shared
// memory), add the noise, pick the k best (score descending, lower expert
// index first on ties) and form the softmax.  Every wait is bounded; on expiry
// the kernel records ST_TIMEOUT, lets copies and MMAs in flight land, writes
// expert -1 and gate 0 for its tokens, frees its tensor memory and exits.
#include "common.cuh"
#include "internal.h"
#include "tmap.h"

#include <atomic>
#include <cstdlib>

namespace moe {

namespace {

constexpr int kRM = 128;                           // tokens per tile (MMA M)
constexpr int kRK = kTmapBoxK;                     // K elements per stage
constexpr int kRThreads = 192;
constexpr int kRMaxStages = 6;
constexpr uint32_t kXTileBytes = kRM * kRK * 2;    // 16 KB of bf16 tokens per stage
constexpr int kRouteTcMaxE = 160;                  // 3 * E_pad <= 512 TMEM columns
constexpr size_t kRouteSmemBudget = 110 * 1024;    // per CTA: two CTAs fit on an SM

// Status word for callers that pass none (moe_route): waits still need one.
__device__ uint32_t g_route_status_scratch;

struct RouteTcArgs {
    const float *W_g;
    const float *b_g;
    const float *noise;
    float sigma;
    int64_t N;
    int d, E, k, stages;
    int splits;  // CTAs per token tile (a cluster), each summing one piece of K
    float *logits_out;
    int32_t *topk_idx;
    float *gates;
    uint32_t *status;  // nullable: the kernel then uses a scratch word of its own
    uint64_t timeout_ns;
};

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// Barrier over the four epilogue warps only (id 1; id 0 is __syncthreads).
__device__ __forceinline__ void epilogue_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ bool wait_until(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > timeout_ns) return false;
    return true;
}

__device__ __forceinline__ bool ranks_before_tc(float v, int e, float v2, int e2) {
    return v > v2 || (v == v2 && e < e2);
}

__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat162 h) {
    return *reinterpret_cast<uint32_t *>(&h);
}

// Three bf16 parts of two fp32 weights (element 0 in the low half).
__device__ __forceinline__ void split3(float a, float b, uint32_t &hi, uint32_t &mid, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const float ra = __fsub_rn(a, hf.x), rb = __fsub_rn(b, hf.y);
    const __nv_bfloat162 m = __floats2bfloat162_rn(ra, rb);
    const float2 mf = __bfloat1622float2(m);
    const __nv_bfloat162 l = __floats2bfloat162_rn(__fsub_rn(ra, mf.x), __fsub_rn(rb, mf.y));
    hi = bf16x2_bits(h);
    mid = bf16x2_bits(m);
    lo = bf16x2_bits(l);
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled K-major tile
// (8-row atoms of 1024 bytes; the chunk index is XORed with the row's phase).
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

template <int UPT>  // E_pad = 16 * UPT experts per part
__host__ __device__ constexpr uint32_t route_tmem_cols() {
    return 3 * 16 * UPT <= 64 ? 64 : 3 * 16 * UPT <= 128 ? 128 : 3 * 16 * UPT <= 256 ? 256 : 512;
}

template <int UPT>
__host__ __device__ constexpr uint32_t route_stage_bytes() {
    return kXTileBytes + 3u * 16u * UPT * kRK * 2u;
}

// Which K blocks CTA `c` of an S-CTA cluster sums: [c*kb/S, (c+1)*kb/S).
__host__ __device__ inline int route_kb_begin(int c, int S, int kb_total) {
    return static_cast<int>(static_cast<int64_t>(c) * kb_total / S);
}

// CTAs per token tile: the K range is cut into S pieces of at least 8 blocks
// (512 columns), S <= 8.  S depends on d only, so a token's logits do not
// depend on the batch size or on where the token sits in the batch.
__host__ __device__ inline int route_k_splits(int d) {
    const int kb_total = (d + kRK - 1) / kRK;
    const int s = (kb_total + 7) / 8;
    return s < 1 ? 1 : (s > 8 ? 8 : s);
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

template <int UPT>
__global__ void __launch_bounds__(kRThreads, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const RouteTcArgs args) {
    constexpr int E_PAD = 16 * UPT;
    constexpr int NB = 3 * E_PAD;                    // rows of B
    constexpr uint32_t STAGE = route_stage_bytes<UPT>();
    constexpr uint32_t TMEM_COLS = route_tmem_cols<UPT>();
    static_assert(STAGE % 1024 == 0, "stage alignment");
    static_assert(NB <= 512, "accumulator columns");

    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t bars[3 * kRMaxStages + 2];
    __shared__ uint32_t tmem_holder;
    __shared__ int epi_fail;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int stages = args.stages;
    const int E = args.E, d = args.d, k = args.k;
    const int kb_total = (d + kRK - 1) / kRK;
    const int S = args.splits;                      // CTAs of this cluster, one K piece each
    const int crank = static_cast<int>(cluster_ctarank());
    const int kb0 = route_kb_begin(crank, S, kb_total), kb1 = route_kb_begin(crank + 1, S, kb_total);
    const int64_t t0 = static_cast<int64_t>(blockIdx.x / S) * kRM;
    const uint64_t tmo = args.timeout_ns;
    uint32_t *status = args.status != nullptr ? args.status : &g_route_status_scratch;

    const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    uint8_t *smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
    const uint32_t xfull0 = smem_u32(&bars[0]);                 // x tile landed (TMA bytes)
    const uint32_t wfull0 = smem_u32(&bars[kRMaxStages]);       // W parts written (4 warps)
    const uint32_t empty0 = smem_u32(&bars[2 * kRMaxStages]);   // MMAs done with the stage
    const uint32_t accf = smem_u32(&bars[3 * kRMaxStages]);     // accumulator final
    const uint32_t drain = smem_u32(&bars[3 * kRMaxStages + 1]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(xfull0 + 8 * s, 1);
            mbar_init(wfull0 + 8 * s, 4);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        fence_barrier_init();
        epi_fail = 0;
    }
    if (warp == 0 && lane == 0) tma_prefetch_desc(&tm_x);
    if (warp == 1) {
        tmem_alloc(smem_u32(&tmem_holder), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // Dependent kernels may start only once every CTA holds its tensor memory,
    // so none of them can take columns this grid still waits for.
    pdl_trigger();
    const uint32_t tmem_base = tmem_holder;
    pdl_wait();
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (x tiles)
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1u, status, tmo, 11)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = xfull0 + 8 * stage;
                mbar_arrive_expect_tx(fb, kXTileBytes);
                tma_load_2d(smem_base + stage * STAGE, &tm_x, fb, kb * kRK, static_cast<int>(t0));
                ++issued;
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                // let copies already in flight land before the CTA can exit
                int st = stage;
                uint32_t ph = phase;
                for (int i = 0; i < stages && i < issued; ++i) {
                    if (st == 0) {
                        st = stages - 1;
                        ph ^= 1u;
                    } else {
                        --st;
                    }
                    wait_until(xfull0 + 8 * st, ph, tmo);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, any = false;
            for (int kb = kb0; kb < kb1 && ok; ++kb) {
                if (!mbar_wait_bounded(xfull0 + 8 * stage, phase, status, tmo, 12) ||
                    !mbar_wait_bounded(wfull0 + 8 * stage, phase, status, tmo, 13)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_base + stage * STAGE;
                const uint64_t ad = smem_desc_sw128(sa);
#pragma unroll
                for (int kk = 0; kk < kRK / 16; ++kk) {
#pragma unroll
                    for (int n0 = 0; n0 < NB; n0 += 256) {
                        constexpr int kChunk = NB < 256 ? NB : 256;
                        const int nn = (NB - n0) < kChunk ? (NB - n0) : kChunk;
                        const uint64_t bd = smem_desc_sw128(sa + kXTileBytes + static_cast<uint32_t>(n0) * 128u);
                        // +32 bytes along K inside the swizzled row = +2 in the address field
                        umma_bf16(tmem_base + static_cast<uint32_t>(n0), ad + 2 * kk, bd + 2 * kk,
                                  idesc_bf16_f32(kRM, nn), (kb > kb0 || kk > 0) ? 1u : 0u);
                    }
                }
                any = true;
                umma_commit(empty0 + 8 * stage);
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) {
                umma_commit(accf);
            } else if (any) {
                umma_commit(drain);
                wait_until(drain, 0, tmo);
            }
        }
    } else {
        // ------------------------------------------------ W_g split, then this K piece's sums
        const int et = threadIdx.x - 64;  // 0..127
        const int q = warp & 3;           // TMEM lane quarter this warp may read
        const int row = q * 32 + lane;
        bool ok = true;
        {
            int stage = 0;
            uint32_t phase = 0;
            for (int kb = kb0; kb < kb1; ++kb) {
                // this K block's weights, loaded before the slot frees up
                float w[UPT][8];
                const int col0 = kb * kRK;
#pragma unroll
                for (int i = 0; i < UPT; ++i) {
                    const int u = et + i * 128;
                    const int e = u >> 3, col = col0 + (u & 7) * 8;
                    if (e < E && col < d) {
                        const float4 *p = reinterpret_cast<const float4 *>(args.W_g + static_cast<int64_t>(e) * d + col);
                        const float4 a = p[0], b = p[1];
                        w[i][0] = a.x; w[i][1] = a.y; w[i][2] = a.z; w[i][3] = a.w;
                        w[i][4] = b.x; w[i][5] = b.y; w[i][6] = b.z; w[i][7] = b.w;
                    } else {
#pragma unroll
                        for (int v = 0; v < 8; ++v) w[i][v] = 0.0f;
                    }
                }
                if (!mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1u, status, tmo, 14)) {
                    ok = false;
                    break;
                }
                uint8_t *bbase = smem_gen + stage * STAGE + kXTileBytes;
#pragma unroll
                for (int i = 0; i < UPT; ++i) {
                    const int u = et + i * 128;
                    const int e = u >> 3, c = u & 7;
                    uint4 hi, mid, lo;
                    split3(w[i][0], w[i][1], hi.x, mid.x, lo.x);
                    split3(w[i][2], w[i][3], hi.y, mid.y, lo.y);
                    split3(w[i][4], w[i][5], hi.z, mid.z, lo.z);
                    split3(w[i][6], w[i][7], hi.w, mid.w, lo.w);
                    *reinterpret_cast<uint4 *>(bbase + sw128_offset(e, c)) = hi;
                    *reinterpret_cast<uint4 *>(bbase + sw128_offset(E_PAD + e, c)) = mid;
                    *reinterpret_cast<uint4 *>(bbase + sw128_offset(2 * E_PAD + e, c)) = lo;
                }
                fence_proxy_async_smem();  // generic-proxy writes -> visible to the MMA
                __syncwarp();
                if (lane == 0) mbar_arrive(wfull0 + 8 * stage);
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // accumulator complete (every MMA, so every read of the ring, is done)
        ok = ok && mbar_wait_bounded(accf, 0, status, tmo, 15);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (ok) {
            // this piece's sum per (token, expert): (hi + mid) + lo, into the
            // partial table [128][ld] that reuses the ring
            const int ld = E + 1 + (E & 1);  // odd row stride: conflict-free column access
            float *part = reinterpret_cast<float *>(smem_gen);
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
            for (int ch = 0; ch < UPT; ++ch) {
                uint32_t h[16], m[16], l[16];
                tmem_ld_32x32b_x16(taddr + ch * 16, h);
                tmem_ld_32x32b_x16(taddr + E_PAD + ch * 16, m);
                tmem_ld_32x32b_x16(taddr + 2 * E_PAD + ch * 16, l);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int e = ch * 16 + i;
                    if (e < E)
                        part[row * ld + e] = __fadd_rn(__fadd_rn(__uint_as_float(h[i]), __uint_as_float(m[i])),
                                                       __uint_as_float(l[i]));
                }
            }
        } else if (lane == 0) {
            epi_fail = 1;
        }
    }
    tc_fence_before();
    cluster_sync();  // every piece's partial table and failure flag is in place

    if (warp >= 2) {
        // ------------------------------------------------ this CTA's token rows
        // CTA c of the cluster finishes rows [c*128/S, (c+1)*128/S) of the tile:
        // adds the S partial sums in piece order, the bias, writes the logits,
        // adds the noise, then picks and normalises.  Its own rows of its own
        // table are read by nobody else, so the final scores go there.
        const int et = threadIdx.x - 64;
        const int ld = E + 1 + (E & 1);
        float *part = reinterpret_cast<float *>(smem_gen);
        const uint32_t part_local = smem_u32(part);
        const uint32_t fail_local = smem_u32(&epi_fail);
        bool good = true;
        for (int c = 0; c < S; ++c) good = good && ld_cluster_s32(map_to_cta(fail_local, c)) == 0;
        const int64_t rows_valid = (args.N - t0) < kRM ? (args.N - t0) : kRM;
        const int r0 = crank * kRM / S;
        int r1 = (crank + 1) * kRM / S;
        if (r1 > rows_valid) r1 = static_cast<int>(rows_valid);
        const int nrows = r1 > r0 ? r1 - r0 : 0;
        const bool use_noise = (args.noise != nullptr) && (args.sigma != 0.0f);
        if (good) {
            const int64_t base = (t0 + r0) * E;
            const int total = nrows * E;
            for (int i = et; i < total; i += 128) {
                const int r = r0 + i / E, e = i % E;
                const uint32_t off = static_cast<uint32_t>(r * ld + e) * 4u;
                float v = ld_cluster_f32(map_to_cta(part_local + off, 0));
                for (int c = 1; c < S; ++c) v = __fadd_rn(v, ld_cluster_f32(map_to_cta(part_local + off, c)));
                if (args.b_g) v = __fadd_rn(v, args.b_g[e]);
                if (args.logits_out) args.logits_out[base + i] = v;
                if (use_noise) v = __fadd_rn(v, __fmul_rn(args.sigma, args.noise[base + i]));
                part[r * ld + e] = v;
            }
        }
        epilogue_sync();
        if (et < nrows) {
            const int r = r0 + et;
            const int64_t t = t0 + r;
            int32_t *ti = args.topk_idx + t * k;
            float *gt = args.gates + t * k;
            if (good) {
                // k rounds: the best score ranked after the previous pick
                const float *sr = part + r * ld;
                float pv = 0.0f;
                int pe = -1;
                for (int j = 0; j < k; ++j) {
                    float bv = 0.0f;
                    int be = -1;
                    for (int e = 0; e < E; ++e) {
                        const float v = sr[e];
                        if ((pe < 0 || ranks_before_tc(pv, pe, v, e)) && (be < 0 || ranks_before_tc(v, e, bv, be))) {
                            bv = v;
                            be = e;
                        }
                    }
                    ti[j] = be;
                    gt[j] = bv;  // the kept score, until the softmax below replaces it
                    pv = bv;
                    pe = be;
                }
                const float mx = gt[0];
                float sum = 0.0f;
                for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, expf(__fsub_rn(gt[j], mx)));
                for (int j = 0; j < k; ++j) gt[j] = __fdiv_rn(expf(__fsub_rn(gt[j], mx)), sum);
            } else {
                for (int j = 0; j < k; ++j) {
                    ti[j] = -1;
                    gt[j] = 0.0f;
                }
            }
        }
    }
    cluster_sync();  // no CTA leaves while another may still read its table
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <int UPT>
cudaError_t launch_route_tc_t(const CUtensorMap &tm, RouteTcArgs a, int64_t tiles, cudaStream_t s) {
    constexpr uint32_t STAGE = route_stage_bytes<UPT>();
    int stages = static_cast<int>((kRouteSmemBudget - 1024) / STAGE);
    if (stages > kRMaxStages) stages = kRMaxStages;
    if (stages < 2) stages = 2;
    const size_t ring = static_cast<size_t>(stages) * STAGE;
    const int ld = a.E + 1 + (a.E & 1);
    if (static_cast<size_t>(kRM) * ld * sizeof(float) > ring) return cudaErrorInvalidValue;
    const size_t smem = ring + 1024;
    a.stages = stages;
    a.splits = route_k_splits(a.d);
    auto kern = route_tc_kernel<UPT>;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::atomic<uint64_t> attr_done{0};  // one bit per device
    const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit == 0 || (attr_done.load() & bit) == 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        attr_done.fetch_or(bit);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * a.splits));
    cfg.blockDim = dim3(kRThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(a.splits);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, tm, a);
}

}  // namespace

bool route_tc_eligible(const void *x, const float *W_g, int64_t N, int d, int E) {
    static const bool enabled = [] {
        const char *v = getenv("MOE_ROUTE_TC");
        return v == nullptr || atoi(v) != 0;
    }();
    return enabled && N > 0 && N < (static_cast<int64_t>(1) << 31) / 8 && d % 8 == 0 && E >= 1 &&
           E <= kRouteTcMaxE && reinterpret_cast<uintptr_t>(x) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(W_g) % 16 == 0;
}

cudaError_t launch_route_tc(const void *x, const float *W_g, const float *b_g, const float *noise, float sigma,
                            int64_t N, int d, int E, int k, float *logits_out, int32_t *topk_idx, float *gates,
                            uint32_t *status, uint64_t timeout_ns, cudaStream_t s) {
    CUtensorMap tm;
    if (!make_tmap_bf16_2d(&tm, x, N, d, kRM)) return cudaErrorInvalidValue;
    RouteTcArgs a{W_g, b_g, noise, sigma, N, d, E, k, 0, 1, logits_out, topk_idx, gates, status, timeout_ns};
    const int64_t tiles = (N + kRM - 1) / kRM;
    if (E <= 16) return launch_route_tc_t<1>(tm, a, tiles, s);
    if (E <= 32) return launch_route_tc_t<2>(tm, a, tiles, s);
    if (E <= 64) return launch_route_tc_t<4>(tm, a, tiles, s);
    if (E <= 96) return launch_route_tc_t<6>(tm, a, tiles, s);
    if (E <= 128) return launch_route_tc_t<8>(tm, a, tiles, s);
    return launch_route_tc_t<10>(tm, a, tiles, s);
}

}  // namespace moe
