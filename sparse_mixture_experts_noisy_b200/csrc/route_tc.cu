// Router on the fifth-generation tensor cores, for bf16 tokens: logits, noise,
// KeepTopK and softmax over the kept scores.
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
// x*w split in three; only the accumulation rounds, in fp32 (tensor memory).
// The three part-sums are added in the order hi, mid, lo.
//
// Tile: 128 tokens (MMA M) x all experts.  B is the 3*E_pad rows
// [w_hi of experts 0..E_pad-1; w_mid ...; w_lo ...] of one 64-wide K block in
// the 128-byte-swizzled K-major layout the MMA reads.  Accumulators: 3*E_pad
// fp32 columns of tensor memory per piece (column c = row c of B).  B comes
// one of two ways:
//   - pre-split: a first small kernel writes the parts of all of W_g, once per
//     call, to a [3*E_pad, d] bf16 scratch, and TMA loads B beside the x tile
//     (the fused forward, which has a workspace);
//   - in-kernel: TMA loads the fp32 W_g tile beside the x tile and four warps
//     split it into the B slot (moe_route, which has none).
// Both give the same B bits, so the same logits.
//
// The K range is cut into S pieces (S depends on d only); each piece is summed
// from zero and the pieces are added in order, so a token's logits do not
// depend on the batch size, on where the token sits, or on which of the two
// kernel forms below ran:
//   - clustered (few tiles): the S CTAs of a cluster each sum one piece of one
//     tile and exchange the sums through distributed shared memory;
//   - persistent (many tiles): one CTA per SM walks whole tiles, each piece in
//     one of up to four tensor-memory buffers, so MMAs and drains overlap.
// Every wait is bounded; on expiry the kernel records ST_TIMEOUT, lets copies
// and MMAs in flight land, writes expert -1 and gate 0 for its tokens, frees
// its tensor memory and exits.
#include "common.cuh"
#include "internal.h"
#include "route_common.cuh"
#include "tmap.h"

#include <atomic>
#include <cstdlib>

namespace moe {

namespace {

using namespace rt;

constexpr int kRMaxStages = 8;
constexpr int kRMaxBuf = 4;                        // persistent form: piece buffers
constexpr int kRouteTcMaxE = 160;                  // 3 * E_pad <= 512 TMEM columns
constexpr int kRouteTcMaxK = 32;                   // pick scratch: k floats per token
constexpr size_t kRouteSmemBudget = 110 * 1024;    // per CTA: two CTAs fit on an SM
constexpr size_t kRpSmemBudget = 225 * 1024;       // per CTA when one fills the SM

// Status word of calls that pass none (moe_route): one per device, read and
// cleared by route_status_read_clear (moe_check_route_status).
__device__ uint32_t g_route_status_scratch;

struct RouteTcArgs {
    const float *b_g;
    const float *noise;
    float sigma;
    int64_t N;
    int d, E, k, stages;
    int splits;    // S: pieces of K
    int pick_off;  // byte offset of the pick scratch: k floats per token row of a tile
    int list_off;  // persistent form with two epilogue groups: byte offset of the pick lists
    float *logits_out;
    int32_t *topk_idx;
    float *gates;
    uint32_t *status;  // nullable: the kernel then reports into the library's own word
    uint64_t timeout_ns;
    int tile_rows;     // tokens per tile (the x box height, <= 128; the rest of the MMA's rows are ignored)
};

// Pre-split of all of W_g: w3[p * E_pad + e][c] = part p of W_g[e][c], zero for
// e >= E.  One thread per 8 columns of one expert row.
__global__ void __launch_bounds__(256)
route_split_kernel(const float *__restrict__ W_g, int E, int E_pad, int d, __nv_bfloat16 *__restrict__ w3) {
    pdl_trigger();
    pdl_wait();
    const int chunks = d / 8;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<int64_t>(E_pad) * chunks) return;
    const int e = static_cast<int>(i / chunks), c = static_cast<int>(i % chunks) * 8;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (e < E) {
        const float4 *p = reinterpret_cast<const float4 *>(W_g + static_cast<int64_t>(e) * d + c);
        a = p[0];
        b = p[1];
    }
    uint4 hi, mid, lo;
    split3(a.x, a.y, hi.x, mid.x, lo.x);
    split3(a.z, a.w, hi.y, mid.y, lo.y);
    split3(b.x, b.y, hi.z, mid.z, lo.z);
    split3(b.z, b.w, hi.w, mid.w, lo.w);
    const int64_t plane = static_cast<int64_t>(E_pad) * d;
    uint4 *o = reinterpret_cast<uint4 *>(w3 + static_cast<int64_t>(e) * d + c);
    o[0] = hi;
    *reinterpret_cast<uint4 *>(w3 + plane + static_cast<int64_t>(e) * d + c) = mid;
    *reinterpret_cast<uint4 *>(w3 + 2 * plane + static_cast<int64_t>(e) * d + c) = lo;
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

// ------------------------------------------------------------------ clustered form
// Cluster of S CTAs per token tile; CTA c sums piece c of K.  Warp roles (192
// threads): warp 0 lane 0 issues the TMA loads into a STAGES-deep ring; warp 1
// owns the tensor memory and its lane 0 issues the MMAs; warps 2-5 split W_g
// into the B slots (in-kernel split only), then write this piece's sums to a
// table in shared memory.  After a cluster barrier CTA c finishes rows
// [c*128/S, (c+1)*128/S) of the tile: adds the S tables in piece order
// (reading the others through distributed shared memory), the bias, writes
// the logits, adds the noise, picks and normalises.
template <int UPT, bool PRE>
__global__ void __launch_bounds__(192, (PRE || UPT <= 2) ? 2 : 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                const RouteTcArgs args) {
    constexpr uint32_t STAGE = route_stage_bytes<UPT, PRE>();
    constexpr uint32_t TMEM_COLS = route_tmem_cols<UPT>();
    static_assert(STAGE % 1024 == 0, "stage alignment");

    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t bars[3 * kRMaxStages + 2];
    __shared__ uint32_t tmem_holder;
    __shared__ int epi_fail;
    __shared__ uint32_t cta_status;  // this CTA's copy of the status word

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int stages = args.stages;
    const int E = args.E, d = args.d, k = args.k;
    const int kb_total = (d + kRK - 1) / kRK;
    const int S = args.splits;
    const int crank = static_cast<int>(cluster_ctarank());
    const int kb0 = route_kb_begin(crank, S, kb_total), kb1 = route_kb_begin(crank + 1, S, kb_total);
    const int64_t t0 = static_cast<int64_t>(blockIdx.x / S) * kRM;
    const uint64_t tmo = args.timeout_ns;
    uint32_t *status = &cta_status;

    const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    uint8_t *smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
    const uint32_t xfull0 = smem_u32(&bars[0]);                 // stage loaded (TMA bytes)
    const uint32_t wfull0 = smem_u32(&bars[kRMaxStages]);       // B slot split (4 warps)
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
        cta_status = 0u;
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
    }
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

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1u, status, tmo, 11)) {
                    ok = false;
                    break;
                }
                load_stage<UPT, PRE>(smem_base + stage * STAGE, &tm_x, &tm_w, xfull0 + 8 * stage, kb,
                                     static_cast<int>(t0), kRM);
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
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!mbar_wait_bounded(xfull0 + 8 * stage, phase, status, tmo, 12) ||
                    (!PRE && !mbar_wait_bounded(wfull0 + 8 * stage, phase, status, tmo, 13))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                mma_stage<UPT>(smem_base + stage * STAGE, tmem_base, kb == kb0);
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
        // ------------------------------------------------ W_g split, then this piece's sums
        const int et = threadIdx.x - 64;  // 0..127
        const int q = warp & 3;           // TMEM lane quarter this warp may read
        const int row = q * 32 + lane;
        bool ok = true;
        if constexpr (!PRE) {
            int stage = 0;
            uint32_t phase = 0;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!mbar_wait_warp(xfull0 + 8 * stage, phase, status, tmo, 14)) {
                    ok = false;
                    break;
                }
                split_stage<UPT>(smem_gen + stage * STAGE, et);
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
        ok = __all_sync(0xffffffffu, ok);
        ok = ok && mbar_wait_warp(accf, 0, status, tmo, 15);
        tc_fence_after();
        if (ok) {
            // this piece's sum per (token, expert) into the table [128][ld]
            // that reuses the ring
            const int ld = E + 1 + (E & 1);  // odd row stride: conflict-free column access
            float *part = reinterpret_cast<float *>(smem_gen);
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
            for (int ch = 0; ch < UPT; ++ch) {
                float p[16];
                piece_chunk<UPT>(taddr, ch, p);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int e = ch * 16 + i;
                    if (e < E) part[row * ld + e] = p[i];
                }
            }
        } else if (lane == 0) {
            epi_fail = 1;
        }
    }
    tc_fence_before();
    cluster_sync();  // every piece's table and failure flag is in place

    if (warp >= 2) {
        // ------------------------------------------------ this CTA's token rows
        // Its own rows of its own table are read by nobody else, so the final
        // scores go there.
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
#pragma unroll 4
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
                pick_row_smem(part + r * ld, E, k, reinterpret_cast<float *>(smem_gen + args.pick_off) + et * k, ti, gt);
            } else {
                for (int j = 0; j < k; ++j) {
                    ti[j] = -1;
                    gt[j] = 0.0f;
                }
            }
        }
    }
    cluster_sync();  // no CTA leaves while another may still read its table
    if (threadIdx.x == 0)
        publish_status(args.status != nullptr ? args.status : &g_route_status_scratch, cta_status);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ persistent form
// One CTA per SM walks tiles tile = blockIdx.x, + gridDim.x, ...; the ring and
// the MMAs run on from one tile to the next.  A tile holds tile_rows tokens
// (at most 128, the MMA's M): the launcher picks it so that every CTA gets the
// same number of tiles, and the MMA rows past tile_rows are computed on
// whatever the stage holds there and never read.  A token's sums do not
// depend on which rows share its tile.  Piece p of the CTA (counting over its
// tiles) sums from zero into tensor-memory buffer p % NBUF; the epilogue adds
// the piece sums in order in registers, so each token gets what the clustered
// form gives it.
//
// Warp roles: warp 0 lane 0 loads stages by TMA; warp 1 owns the tensor
// memory and its lane 0 issues the MMAs; an epilogue group of four warps
// drains the accumulators (one token row per thread) and finishes a tile
// (bias, logits, noise, KeepTopK, softmax).  With pre-split weights and
// E_pad = 32 or 64, warps 2-5 and 6-9 are two epilogue groups that both drain
// every piece, group g for the experts [g E_pad/2, (g+1) E_pad/2): each picks
// the top k of its half, and group 0 merges the two pick lists (320 threads,
// 168 registers a thread).  With the in-kernel split, warps 2-5 are the one
// group and warps 6-9 split W_g into the B slots; E_pad = 16 or 80 with
// pre-split weights runs one group in 192 threads.
template <int UPT, bool PRE>
__host__ __device__ constexpr int routep_groups() {
    return (PRE && (UPT == 2 || UPT == 4)) ? 2 : 1;
}

// Barrier over the eight epilogue warps (id 2).
__device__ __forceinline__ void epilogue_pair_sync() { asm volatile("bar.sync 2, 256;" ::: "memory"); }
template <int UPT, bool PRE>
__host__ __device__ constexpr int routep_threads() {
    return 64 + 128 * routep_groups<UPT, PRE>() + (PRE ? 0 : 128);
}

template <int UPT, bool PRE>
__global__ void __launch_bounds__(routep_threads<UPT, PRE>(), 1)
route_tcp_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                 const RouteTcArgs args) {
    constexpr int ACC = route_acc_cols<UPT>();
    constexpr int NBUF = routep_nbuf<UPT>();
    constexpr int NG = routep_groups<UPT, PRE>();
    constexpr int NCH = UPT / NG;  // 16-expert chunks one epilogue thread handles
    constexpr int HE = 16 * NCH;
    static_assert(NCH * NG == UPT, "the groups split the chunks evenly");
    constexpr uint32_t STAGE = route_stage_bytes<UPT, PRE>();
    constexpr uint32_t TMEM_COLS = routep_tmem_cols<UPT>();
    static_assert(NBUF >= 2 && NBUF <= kRMaxBuf, "piece buffers");
    static_assert(STAGE % 1024 == 0, "stage alignment");

    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t bars[3 * kRMaxStages + 2 * kRMaxBuf + 1];
    __shared__ uint32_t tmem_holder;
    __shared__ uint32_t cta_status;  // this CTA's copy of the status word

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int stages = args.stages;
    const int E = args.E, d = args.d, k = args.k;
    const int kb_total = (d + kRK - 1) / kRK;
    const int S = args.splits;
    const int tile_rows = args.tile_rows;
    const int64_t tiles = (args.N + tile_rows - 1) / tile_rows;
    const uint64_t tmo = args.timeout_ns;
    uint32_t *status = &cta_status;

    const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    uint8_t *smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
    const uint32_t xfull0 = smem_u32(&bars[0]);
    const uint32_t wfull0 = smem_u32(&bars[kRMaxStages]);
    const uint32_t empty0 = smem_u32(&bars[2 * kRMaxStages]);
    const uint32_t accf0 = smem_u32(&bars[3 * kRMaxStages]);             // [NBUF] piece sum ready
    const uint32_t acce0 = smem_u32(&bars[3 * kRMaxStages + kRMaxBuf]);  // [NBUF] buffer drained
    const uint32_t drain = smem_u32(&bars[3 * kRMaxStages + 2 * kRMaxBuf]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(xfull0 + 8 * s, 1);
            mbar_init(wfull0 + 8 * s, 4);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(accf0 + 8 * b, 1);
            mbar_init(acce0 + 8 * b, 4 * NG);  // every epilogue warp
        }
        mbar_init(drain, 1);
        fence_barrier_init();
        cta_status = 0u;
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tmem_holder), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_trigger();  // after the tensor memory is held (see the clustered form)
    const uint32_t tmem_base = tmem_holder;
    pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                for (int kb = 0; kb < kb_total; ++kb) {
                    if (!mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1u, status, tmo, 21)) {
                        ok = false;
                        break;
                    }
                    load_stage<UPT, PRE>(smem_base + stage * STAGE, &tm_x, &tm_w, xfull0 + 8 * stage, kb,
                                         static_cast<int>(tile * tile_rows), tile_rows);
                    ++issued;
                    if (++stage == stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
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
            int piece = 0;  // pieces issued by this CTA so far
            bool ok = true, any = false;
            for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                for (int c = 0; c < S && ok; ++c, ++piece) {
                    const int b = piece % NBUF;
                    const uint32_t use = static_cast<uint32_t>(piece / NBUF);
                    if (!mbar_wait_bounded(acce0 + 8 * b, (use & 1u) ^ 1u, status, tmo, 22)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int kb0 = route_kb_begin(c, S, kb_total), kb1 = route_kb_begin(c + 1, S, kb_total);
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * ACC);
                    for (int kb = kb0; kb < kb1; ++kb) {
                        if (!mbar_wait_bounded(xfull0 + 8 * stage, phase, status, tmo, 23) ||
                            (!PRE && !mbar_wait_bounded(wfull0 + 8 * stage, phase, status, tmo, 24))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        mma_stage<UPT>(smem_base + stage * STAGE, d_tmem, kb == kb0);
                        any = true;
                        umma_commit(empty0 + 8 * stage);
                        if (++stage == stages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (ok) umma_commit(accf0 + 8 * b);
                }
            }
            if (!ok && any) {
                umma_commit(drain);
                wait_until(drain, 0, tmo);
            }
        }
    } else if (!PRE && warp >= 6) {
        // ------------------------------------------------ W_g split into the B slots
        if constexpr (!PRE) {
            const int et = threadIdx.x - 192;  // 0..127
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                for (int kb = 0; kb < kb_total; ++kb) {
                    if (!mbar_wait_warp(xfull0 + 8 * stage, phase, status, tmo, 25)) {
                        ok = false;
                        break;
                    }
                    split_stage<UPT>(smem_gen + stage * STAGE, et);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(wfull0 + 8 * stage);
                    if (++stage == stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue group g (warps 2-5, 6-9)
        // Group g drains and finishes the experts [g HE, (g + 1) HE) of every
        // token of every tile (one token row per thread).
        const int g = (warp - 2) >> 2;
        const int q = warp & 3;  // TMEM lane quarter
        const int row = q * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const int e0 = g * HE;
        float *pv = reinterpret_cast<float *>(smem_gen + args.pick_off) + row * k;  // [128][k] kept scores
        const bool use_noise = (args.noise != nullptr) && (args.sigma != 0.0f);
        const bool vec4 = (E & 3) == 0;  // rows of E floats are 16-byte aligned
        bool ok = true;
        int piece = 0, tt = 0;
        for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tt) {
            const int64_t t = tile * tile_rows + row;
            const bool mine = row < tile_rows && t < args.N;
            float run[HE];
            float eps[NG == 2 ? HE : 1];  // this token's noise (its part), loaded while the last piece's MMAs run
            for (int c = 0; c < S; ++c, ++piece) {
                if constexpr (NG == 2) {
                  if (c == S - 1 && use_noise && mine) {
                    const float *nz = args.noise + t * E + e0;
#pragma unroll
                    for (int e = 0; e < HE; e += 4) {
                        if (vec4) {
                            if (e0 + e < E) {
                                const float4 f = *reinterpret_cast<const float4 *>(nz + e);
                                eps[e] = f.x; eps[e + 1] = f.y; eps[e + 2] = f.z; eps[e + 3] = f.w;
                            }
                        } else {
#pragma unroll
                            for (int v = 0; v < 4; ++v)
                                if (e0 + e + v < E) eps[e + v] = nz[e + v];
                        }
                    }
                  }
                }
                const int b = piece % NBUF;
                const uint32_t use = static_cast<uint32_t>(piece / NBUF);
                ok = __all_sync(0xffffffffu, ok);
                if (ok) ok = mbar_wait_warp(accf0 + 8 * b, use & 1u, status, tmo, 26);
                tc_fence_after();
                if (ok)
                    drain_piece<UPT, NCH>(tmem_base + lane_off + static_cast<uint32_t>(b * ACC), c == 0, run, g * NCH);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acce0 + 8 * b);
            }
            // finish this thread's part of the token: bias, logits out, noise
            if (mine && ok) {
                if (args.b_g) {
#pragma unroll
                    for (int e = 0; e < HE; ++e)
                        if (e0 + e < E) run[e] = __fadd_rn(run[e], args.b_g[e0 + e]);
                }
                if (args.logits_out) {
                    float *lo = args.logits_out + t * E + e0;
#pragma unroll
                    for (int e = 0; e < HE; e += 4) {
                        if (vec4) {
                            if (e0 + e < E)
                                *reinterpret_cast<float4 *>(lo + e) = make_float4(run[e], run[e + 1], run[e + 2], run[e + 3]);
                        } else {
#pragma unroll
                            for (int v = 0; v < 4; ++v)
                                if (e0 + e + v < E) lo[e + v] = run[e + v];
                        }
                    }
                }
                if (use_noise) {
                    if constexpr (NG == 1) {
                        const float *nz = args.noise + t * E;
#pragma unroll
                        for (int e = 0; e < HE; e += 4) {
                            float q4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                            if (vec4) {
                                if (e < E) {
                                    const float4 f = *reinterpret_cast<const float4 *>(nz + e);
                                    q4[0] = f.x; q4[1] = f.y; q4[2] = f.z; q4[3] = f.w;
                                }
                            } else {
#pragma unroll
                                for (int v = 0; v < 4; ++v)
                                    if (e + v < E) q4[v] = nz[e + v];
                            }
#pragma unroll
                            for (int v = 0; v < 4; ++v)
                                if (e + v < E) run[e + v] = __fadd_rn(run[e + v], __fmul_rn(args.sigma, q4[v]));
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < HE; ++e)
                            if (e0 + e < E) run[e] = __fadd_rn(run[e], __fmul_rn(args.sigma, eps[e]));
                    }
                }
            }
            // KeepTopK and softmax
            int32_t *ti = args.topk_idx + t * k;
            float *gt = args.gates + t * k;
            if constexpr (NG == 1) {
                if (mine) {
                    if (ok) {
                        pick_row_regs<HE>(run, E, k, pv, ti, gt);
                    } else {
                        for (int j = 0; j < k; ++j) {
                            ti[j] = -1;
                            gt[j] = 0.0f;
                        }
                    }
                }
            } else {
                // each part's picks in pick order: part 0 to list 0, part 1 to list
                // 1 or 2 by tile parity (part 0 of the next tile cannot be merged
                // before this barrier of the next tile, so list 1 / 2 is free by
                // the time part 1 writes it again)
                uint32_t *lw = reinterpret_cast<uint32_t *>(smem_gen + args.list_off);  // [3][128][k]
                int32_t *li = reinterpret_cast<int32_t *>(lw + 3 * kRM * k);            // [3][128][k]
                const int list = g == 0 ? 0 : 1 + (tt & 1);
                if (mine && ok)
                    pick_part_regs<HE>(run, e0, E, k, lw + (list * kRM + row) * k, li + (list * kRM + row) * k);
                epilogue_pair_sync();
                if (g == 0 && mine) {
                    const int other = 1 + (tt & 1);
                    const bool good = ok && (*reinterpret_cast<volatile uint32_t *>(status) & ST_ABORT) == 0u;
                    if (good) {
                        merge_picks(lw + row * k, li + row * k, lw + (other * kRM + row) * k,
                                    li + (other * kRM + row) * k, k, pv, ti);
                        softmax_kept(pv, k, gt);
                    } else {
                        for (int j = 0; j < k; ++j) {
                            ti[j] = -1;
                            gt[j] = 0.0f;
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0)
        publish_status(args.status != nullptr ? args.status : &g_route_status_scratch, cta_status);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// The persistent form keeps a token's E_pad running sums and its pick words
// in registers: E_pad <= 64 at 320 threads (168 registers a thread), and
// E_pad = 80 with pre-split weights at 192 threads.
__host__ __device__ constexpr bool route_persistent_ok(int upt, bool pre) {
    return upt <= 4 || (upt == 5 && pre);
}

template <int UPT, bool PRE, int KIND>  // KIND: 0 clustered, 1 persistent
cudaError_t set_smem_attr(void (*kern)(CUtensorMap, CUtensorMap, RouteTcArgs), size_t smem) {
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
    return cudaSuccess;
}

template <int UPT, bool PRE>
cudaError_t launch_cluster_t(const CUtensorMap &tm, const CUtensorMap &tw, RouteTcArgs a, int64_t tiles, int sms,
                             cudaStream_t s) {
    constexpr uint32_t STAGE = route_stage_bytes<UPT, PRE>();
    // a grid that fits on the SMs at once: one CTA per SM with every stage it
    // can hold (a piece's K blocks all in flight); else two CTAs per SM when
    // two stages fit the half budget, else one CTA with as many stages as fit
    const bool one_wave = tiles * a.splits <= sms;
    const size_t budget =
        (!one_wave && 2 * STAGE + 1024 <= kRouteSmemBudget) ? kRouteSmemBudget : kRpSmemBudget;
    int stages = static_cast<int>((budget - 1024) / STAGE);
    if (stages > kRMaxStages) stages = kRMaxStages;
    if (stages < 1) return cudaErrorInvalidValue;
    const size_t ring = static_cast<size_t>(stages) * STAGE;
    const int ld = a.E + 1 + (a.E & 1);
    const size_t part_bytes = align_up(static_cast<size_t>(kRM) * ld * sizeof(float), 16);
    if (part_bytes + static_cast<size_t>(kRM) * a.k * sizeof(float) > ring) return cudaErrorInvalidValue;
    const size_t smem = ring + 1024;
    a.stages = stages;
    a.pick_off = static_cast<int>(part_bytes);
    auto kern = route_tc_kernel<UPT, PRE>;
    // the attribute is set once per device: to the largest request of any form
    cudaError_t e = set_smem_attr<UPT, PRE, 0>(kern, kRpSmemBudget);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * a.splits));
    cfg.blockDim = dim3(192);
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
    return cudaLaunchKernelEx(&cfg, kern, tm, tw, a);
}

template <int UPT, bool PRE>
cudaError_t launch_persistent_t(const CUtensorMap &tm, const CUtensorMap &tw, RouteTcArgs a, int64_t tiles,
                                int sms, cudaStream_t s) {
    constexpr uint32_t STAGE = route_stage_bytes<UPT, PRE>();
    // kept scores [128][k] floats, then (two groups) the pick lists: words
    // and indices [3][128][k] each
    const size_t pick_bytes = static_cast<size_t>(kRM) * a.k * sizeof(float);
    const size_t list_bytes =
        routep_groups<UPT, PRE>() == 2 ? 2 * 3 * static_cast<size_t>(kRM) * a.k * sizeof(uint32_t) : 0;
    const size_t fixed = pick_bytes + list_bytes + 1024;
    if (fixed + STAGE > kRpSmemBudget) return cudaErrorInvalidValue;
    int stages = static_cast<int>((kRpSmemBudget - fixed) / STAGE);
    if (stages > kRMaxStages) stages = kRMaxStages;
    const size_t ring = static_cast<size_t>(stages) * STAGE;
    const size_t smem = ring + fixed;
    a.stages = stages;
    a.pick_off = static_cast<int>(ring);
    a.list_off = static_cast<int>(ring + pick_bytes);
    auto kern = route_tcp_kernel<UPT, PRE>;
    cudaError_t e = set_smem_attr<UPT, PRE, 1>(kern, kRpSmemBudget);  // once per device: the largest request
    if (e != cudaSuccess) return e;
    const int64_t grid = tiles < sms ? tiles : sms;
    return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(routep_threads<UPT, PRE>()), smem, s, tm, tw, a);
}

template <int UPT, bool PRE>
cudaError_t launch_form(bool persistent, const CUtensorMap &tm, const CUtensorMap &tw, const RouteTcArgs &a,
                        int64_t tiles, int sms, cudaStream_t s) {
    if constexpr (route_persistent_ok(UPT, PRE) && routep_nbuf<UPT>() >= 2) {
        if (persistent) return launch_persistent_t<UPT, PRE>(tm, tw, a, tiles, sms, s);
    }
    return launch_cluster_t<UPT, PRE>(tm, tw, a, tiles, sms, s);
}

template <bool PRE>
cudaError_t launch_upt(int upt, bool persistent, const CUtensorMap &tm, const CUtensorMap &tw, const RouteTcArgs &a,
                       int64_t tiles, int sms, cudaStream_t s) {
    switch (upt) {
        case 1: return launch_form<1, PRE>(persistent, tm, tw, a, tiles, sms, s);
        case 2: return launch_form<2, PRE>(persistent, tm, tw, a, tiles, sms, s);
        case 4: return launch_form<4, PRE>(persistent, tm, tw, a, tiles, sms, s);
        case 5: return launch_form<5, PRE>(persistent, tm, tw, a, tiles, sms, s);
        case 6: return launch_form<6, PRE>(persistent, tm, tw, a, tiles, sms, s);
        case 8: return launch_form<8, PRE>(persistent, tm, tw, a, tiles, sms, s);
        case 10: return launch_form<10, PRE>(persistent, tm, tw, a, tiles, sms, s);
        default: return cudaErrorInvalidValue;
    }
}

// E_pad / 16 for E experts: the same value everywhere a given E is routed.
int route_upt(int E) {
    return E <= 16 ? 1 : E <= 32 ? 2 : E <= 64 ? 4 : E <= 80 ? 5 : E <= 96 ? 6 : E <= 128 ? 8 : 10;
}

// MOE_ROUTE_TCP=0 keeps large batches on the clustered form (for comparisons).
bool route_tcp_enabled() {
    static const bool enabled = [] {
        const char *v = getenv("MOE_ROUTE_TCP");
        return v == nullptr || atoi(v) != 0;
    }();
    return enabled;
}

}  // namespace

// Whether a call with a pre-split workspace reads the split weights: only the
// persistent form does.  The clustered form (few tiles) splits W_g in-kernel,
// which gives the same bits and saves the split kernel's launch.
bool route_tc_presplit_used(int64_t N, int d, int E, int sms) {
    const int64_t tiles = (N + kRM - 1) / kRM;
    return tiles * route_k_splits(d) >= 2 * static_cast<int64_t>(sms) && route_tcp_enabled() &&
           route_persistent_ok(route_upt(E), true);
}

bool route_tc_shape_ok(int64_t N, int d, int E, int k) {
    static const bool enabled = [] {
        const char *v = getenv("MOE_ROUTE_TC");
        return v == nullptr || atoi(v) != 0;
    }();
    return enabled && N > 0 && N < (static_cast<int64_t>(1) << 31) / 8 && d % 8 == 0 && E >= 1 &&
           E <= kRouteTcMaxE && k >= 1 && k <= kRouteTcMaxK;
}

bool route_tc_eligible(const void *x, const float *W_g, int64_t N, int d, int E, int k) {
    return route_tc_shape_ok(N, d, E, k) && reinterpret_cast<uintptr_t>(x) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(W_g) % 16 == 0;
}

size_t route_tc_w3_bytes(int d, int E) {
    if (d < 1 || d % 8 != 0 || E < 1 || E > kRouteTcMaxE) return 0;
    return align_up(static_cast<size_t>(3) * 16 * route_upt(E) * d * 2, 256);
}

cudaError_t launch_route_tc(const void *x, const float *W_g, const float *b_g, const float *noise, float sigma,
                            int64_t N, int d, int E, int k, float *logits_out, int32_t *topk_idx, float *gates,
                            uint32_t *status, uint64_t timeout_ns, void *w3, cudaStream_t s) {
    CUtensorMap tm, tw;
    const int upt = route_upt(E);
    const int e_pad = 16 * upt, nb = 3 * e_pad;
    static_assert(routep_nbuf<5>() >= 2 && !route_persistent_ok(6, true), "persistent forms");
    RouteTcArgs a{b_g, noise, sigma, N, d, E, k, 0, route_k_splits(d), 0, 0, logits_out, topk_idx, gates, status,
                  timeout_ns, kRM};
    int64_t tiles = (N + kRM - 1) / kRM;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (w3 != nullptr && !route_tc_presplit_used(N, d, E, sms)) w3 = nullptr;
    // many tiles: the persistent form; few: clusters spread one tile's K over
    // up to 8 SMs
    // (the persistent form holds up to 64, or 80 with pre-split weights,
    // experts' sums in registers)
    const bool persistent = tiles * a.splits >= 2 * static_cast<int64_t>(sms) && route_tcp_enabled() &&
                            route_persistent_ok(upt, w3 != nullptr);
    if (persistent) {
        // the same number of tiles on every SM: waves of full tiles, then the
        // tile height that spreads N evenly over that many waves
        const int64_t waves = (tiles + sms - 1) / sms;
        const int64_t rows = (N + waves * sms - 1) / (waves * sms);
        a.tile_rows = static_cast<int>(rows < 8 ? 8 : rows);
        tiles = (N + a.tile_rows - 1) / a.tile_rows;
    }
    if (!make_tmap_bf16_2d(&tm, x, N, d, a.tile_rows)) return cudaErrorInvalidValue;
    if (w3 != nullptr) {
        // the parts of all of W_g, then B by TMA
        const int64_t units = static_cast<int64_t>(e_pad) * (d / 8);
        cudaError_t e = launch_pdl(route_split_kernel, dim3(static_cast<unsigned>((units + 255) / 256)), dim3(256), 0,
                                   s, W_g, E, e_pad, d, static_cast<__nv_bfloat16 *>(w3));
        if (e != cudaSuccess) return e;
        if (!make_tmap_bf16_2d(&tw, w3, nb, d, nb <= 256 ? nb : nb / 2)) return cudaErrorInvalidValue;
    } else {
        if (!make_tmap_f32_2d(&tw, W_g, E, d, e_pad, kRK)) return cudaErrorInvalidValue;
    }
    return w3 != nullptr ? launch_upt<true>(upt, persistent, tm, tw, a, tiles, sms, s)
                         : launch_upt<false>(upt, persistent, tm, tw, a, tiles, sms, s);
}

cudaError_t route_status_read_clear(uint32_t *word, cudaStream_t s) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(word, g_route_status_scratch, sizeof(uint32_t), 0,
                                              cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    const uint32_t zero = 0u;
    e = cudaMemcpyToSymbolAsync(g_route_status_scratch, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(s);
}

}  // namespace moe
