// The whole layer for a small batch (decode: at most 64 tokens) in one
// persistent, cooperative launch: router, slot assignment, gather, the two
// weight-streaming expert GEMMs and the combine.
//
// "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 1-12 (one
// token's way through the layer: logits, noise, KeepTopK, softmax, dispatch,
// W_up, ReLU, W_down, gate scaling, sum); "nanoMoEの深層解剖" slides 11-40.
//
// At 64 tokens the layer's time is the time to stream every touched expert's
// weights once (1.88 GB at the Mixtral shape).  Run as separate kernels, the
// router, the slot pass and the gather come first and HBM idles meanwhile.
// Here the weight tiles of each CTA's first GEMM units are loaded into its
// shared-memory ring from the start: a weight tile does not depend on the
// routing, only the token tile beside it does, so each ring stage is filled
// in two halves on a barrier that expects two arrivals, and the token half
// is issued once the gathered rows exist.
//
// Phases, with grid-wide counters in the workspace between them (every CTA is
// resident, which the cooperative launch guarantees, and every wait is
// bounded in time):
//   1. router: CTAs 0..S-1 each sum one K piece of the 128-row token tile on
//      the tensor cores, exactly as the router kernels do (route_common.cuh),
//      and publish the piece table;
//   2. CTA 0 adds the pieces, bias and noise, picks the top k, forms the gates
//      and assigns the slots (all first choices before all second choices,
//      capacity cut), then raises a flag;
//   3. every CTA gathers its share of the kept rows;
//   4. up projection: weight-row tiles x the expert's tokens, K split into
//      fp32 partials;
//   5. every CTA sums its share of the partials, applies ReLU and rounds H;
//   6. down projection, K split into fp32 partials;
//   7. combine: each token's partials summed in split order, gate-weighted
//      in choice order.
// Each step does the same arithmetic in the same order as the separate
// kernels of the decode plan, so the output equals theirs bit for bit.
#include "common.cuh"
#include "internal.h"
#include "route_common.cuh"
#include "tmap.h"

namespace moe {

namespace {

using namespace rt;

constexpr int kFThreads = 192;
constexpr int kFStages = 8;
constexpr int kFBN = 64;                                    // tokens of one expert (MMA N, at most)
constexpr uint32_t kFWBytes = 128u * kRK * 2u;              // weight tile: 128 rows x 64 K
constexpr uint32_t kFTBytes = static_cast<uint32_t>(kFBN) * kRK * 2u;  // token tile: 64 rows x 64 K
constexpr uint32_t kFRouteBytes = route_stage_bytes<1, false>();       // x tile + B slot + fp32 W_g tile
constexpr uint32_t kFSlot = kFRouteBytes > kFWBytes + kFTBytes ? kFRouteBytes : kFWBytes + kFTBytes;
static_assert(kFSlot % 1024 == 0, "slot alignment");
constexpr uint32_t kFTmemCols = 256;   // [0, 128): two GEMM accumulators; [128, 176): the router piece
constexpr uint32_t kFRouteCol = 128;
constexpr int kFMaxK = 32;

// Grid-wide counters (workspace words, zero at launch).
enum { SY_PIECES = 0, SY_ROUTED, SY_GATHERED, SY_UP, SY_H, SY_DOWN, SY_ABORT, SY_WORDS };

struct FusedArgs {
    const __nv_bfloat16 *x;
    const float *b_g, *noise;
    float sigma;
    int N, d, E, k, d_ff;
    int64_t C;
    int S;            // router K pieces
    int s_up, s_dn;   // K splits of the two projections
    float *logits_out;
    int32_t *topk, *slot, *counts, *offsets;
    float *gates;
    __nv_bfloat16 *xg, *H, *y;
    float *parts_up, *parts_dn;  // [s_up][rows][d_ff], [s_dn][rows][d]
    int64_t up_stride, dn_stride;
    float *pieces;               // [S][N][E]
    uint32_t *sync;              // SY_WORDS words
    uint32_t *status;
    uint64_t timeout_ns;
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Waits until the counter reaches `target`, for at most timeout_ns; gives up
// early if another CTA raised the abort word.  On expiry it raises the abort
// word and records ST_TIMEOUT with `where` in the CTA's status copy.
__device__ __forceinline__ bool wait_count(const FusedArgs &a, int which, uint32_t target, uint32_t *cta_status,
                                           uint32_t where) {
    const uint32_t *p = a.sync + which;
    if (ld_acquire_u32(p) >= target) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (ld_acquire_u32(p) >= target) return true;
        if (ld_acquire_u32(a.sync + SY_ABORT) != 0u) return false;
        if (global_timer_ns() - t0 > a.timeout_ns) {
            atomicExch(a.sync + SY_ABORT, 1u);
            atomicOr(cta_status, ST_TIMEOUT | ST_ABORT | ((where & 0xFFu) << ST_WHERE_SHIFT));
            return false;
        }
        __nanosleep(256);
    }
}

// The 128 threads of warps 2-5 synchronise only through the helpers below,
// which every one of them calls the same number of times; a thread that
// meets a failure sets *fail_s, and all of them read it after each barrier.
//
// Publish: barrier, then one thread fences and adds 1 to the counter (it adds
// even after a failure, so that no other CTA waits in vain).
__device__ __forceinline__ bool epi_arrive(const FusedArgs &a, int which, int et, const int *fail_s) {
    fence_proxy_async_global();  // generic writes that TMA loads will read
    epilogue_sync();
    if (et == 0) {
        __threadfence();
        atomicAdd(a.sync + which, 1u);
    }
    return *reinterpret_cast<const volatile int *>(fail_s) == 0;
}

// Wait for a counter (one thread polls), then barrier; false if this CTA or
// the layer gave up.
__device__ __forceinline__ bool epi_wait(const FusedArgs &a, int which, uint32_t target, int et,
                                         uint32_t *cta_status, uint32_t where, int *fail_s) {
    if (et == 0 && *reinterpret_cast<volatile int *>(fail_s) == 0 &&
        !wait_count(a, which, target, cta_status, where))
        *fail_s = 1;
    epilogue_sync();
    __threadfence();
    return *reinterpret_cast<const volatile int *>(fail_s) == 0;
}

// One GEMM unit of the fixed enumeration (no counts needed): expert e,
// weight rows w0.., K blocks [kb0, kb1), split index.
struct FUnit {
    int e, w0, kb0, kb1, split;
};
__device__ __forceinline__ FUnit f_unit(int u, int Nw, int K, int splits) {
    const int mt = (Nw + 127) / 128;
    const int kbt = (K + kRK - 1) / kRK;
    FUnit t;
    t.e = u / (mt * splits);
    const int r = u - t.e * (mt * splits);
    t.split = r % splits;
    t.w0 = (r / splits) * 128;
    t.kb0 = static_cast<int>(static_cast<int64_t>(t.split) * kbt / splits);
    t.kb1 = static_cast<int>(static_cast<int64_t>(t.split + 1) * kbt / splits);
    return t;
}

__global__ void __launch_bounds__(kFThreads, 1)
decode_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wg,
                    const __grid_constant__ CUtensorMap tm_wup, const __grid_constant__ CUtensorMap tm_wdn,
                    const __grid_constant__ CUtensorMap tm_xg, const __grid_constant__ CUtensorMap tm_h,
                    const FusedArgs a) {
    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t bars[4 * kFStages + 6];
    __shared__ uint32_t tmem_holder;
    __shared__ uint32_t cta_status;
    __shared__ int fail_s;  // warps 2-5: some thread of this CTA gave up
    __shared__ float pick_s[kFBN * kFMaxK];
    __shared__ int32_t sl_tot[16], sl_w0[16], sl_off[17];
    // counts and offsets of the routing, copied once by the producer when the
    // gathered rows exist (read by the producer and, after a stage's barrier,
    // by the MMA lane: no global load on their per-stage paths)
    __shared__ int32_t cnt_sm[16], off_sm[16];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, b = blockIdx.x;
    const int E = a.E, k = a.k, N = a.N, d = a.d, d_ff = a.d_ff;
    const bool router_cta = b < a.S;
    const int kbt_r = (d + kRK - 1) / kRK;
    const int rkb0 = router_cta ? route_kb_begin(b, a.S, kbt_r) : 0;
    const int rkb1 = router_cta ? route_kb_begin(b + 1, a.S, kbt_r) : 0;
    const int units_up = E * ((d_ff + 127) / 128) * a.s_up;
    const int units_dn = E * ((d + 127) / 128) * a.s_dn;
    uint32_t *status = &cta_status;
    const uint64_t tmo = a.timeout_ns;

    const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    uint8_t *smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
    const uint32_t empty0 = smem_u32(&bars[0]);               // [stages] MMAs done with the slot
    const uint32_t gfull0 = smem_u32(&bars[kFStages]);        // [stages] weight half + token half
    const uint32_t rfull0 = smem_u32(&bars[2 * kFStages]);    // [stages] router stage loaded
    const uint32_t rsplit0 = smem_u32(&bars[3 * kFStages]);   // [stages] W_g split (4 warps)
    const uint32_t tfull0 = smem_u32(&bars[4 * kFStages]);    // [2]
    const uint32_t tempty0 = smem_u32(&bars[4 * kFStages + 2]);  // [2]
    const uint32_t racc = smem_u32(&bars[4 * kFStages + 4]);
    const uint32_t drain = smem_u32(&bars[4 * kFStages + 5]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFStages; ++s) {
            mbar_init(empty0 + 8 * s, 1);
            mbar_init(gfull0 + 8 * s, 2);
            mbar_init(rfull0 + 8 * s, 1);
            mbar_init(rsplit0 + 8 * s, 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(tfull0 + 8 * i, 1);
            mbar_init(tempty0 + 8 * i, 4);
        }
        mbar_init(racc, 1);
        mbar_init(drain, 1);
        fence_barrier_init();
        cta_status = 0u;
        fail_s = 0;
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_wg);
        tma_prefetch_desc(&tm_wup);
        tma_prefetch_desc(&tm_wdn);
        tma_prefetch_desc(&tm_xg);
        tma_prefetch_desc(&tm_h);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tmem_holder), kFTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int slot = 0;
            uint32_t ephase = 0, gpar = 0, rpar = 0;
            bool ok = true;
            // router stages (router CTAs only)
            for (int kb = rkb0; kb < rkb1 && ok; ++kb) {
                if (!mbar_wait_bounded(empty0 + 8 * slot, ephase ^ 1u, status, tmo, 41)) {
                    ok = false;
                    break;
                }
                const uint32_t st = smem_base + slot * kFSlot;
                const uint32_t fb = rfull0 + 8 * slot;
                mbar_arrive_expect_tx(fb, kXTileBytes + route_wtile_bytes<1, false>());
                tma_load_2d(st, &tm_x, fb, kb * kRK, 0);
                tma_load_2d(st + kXTileBytes + route_b_bytes<1>(), &tm_wg, fb, kb * kRK, 0);
                rpar ^= 1u << slot;
                if (++slot == kFStages) {
                    slot = 0;
                    ephase ^= 1u;
                }
            }
            // GEMM stages: weight halves run ahead; token halves follow once
            // the rows they read exist.  A FIFO of the stages whose token half
            // is still owed (at most the ring's depth).
            int pend_slot[kFStages] = {}, pend_e[kFStages] = {}, pend_kb[kFStages] = {}, pend_dn[kFStages] = {};
            int ph = 0, pt = 0;  // FIFO head / tail (counts)
            bool gathered = false, hready = false;
            auto issue_token = [&](int i) -> bool {
                const int q = i % kFStages;
                const bool dn = pend_dn[q] != 0;
                bool &ready = dn ? hready : gathered;
                if (!ready) {
                    if (!wait_count(a, dn ? SY_H : SY_GATHERED, static_cast<uint32_t>(G), status, dn ? 43 : 42))
                        return false;
                    fence_proxy_async_global();
                    ready = true;
                    if (!dn) {  // up stages come first: the routing is final from here on
                        for (int e2 = 0; e2 < E; ++e2) {
                            cnt_sm[e2] = *reinterpret_cast<volatile const int32_t *>(a.counts + e2);
                            off_sm[e2] = *reinterpret_cast<volatile const int32_t *>(a.offsets + e2);
                        }
                    }
                }
                const int e = pend_e[q];
                const uint32_t fb = gfull0 + 8 * pend_slot[q];
                const int cnt = cnt_sm[e];
                if (cnt > 0) {
                    const int row0 = off_sm[e];
                    mbar_arrive_expect_tx(fb, kFTBytes);
                    tma_load_2d(smem_base + pend_slot[q] * kFSlot + kFWBytes, dn ? &tm_h : &tm_xg, fb,
                                pend_kb[q] * kRK, row0);
                } else {
                    mbar_arrive(fb);  // no tokens: the MMA warp only releases the slot
                }
                return true;
            };
            for (int phase = 0; phase < 2 && ok; ++phase) {
                const int units = phase == 0 ? units_up : units_dn;
                const int Nw = phase == 0 ? d_ff : d, K = phase == 0 ? d : d_ff;
                const int splits = phase == 0 ? a.s_up : a.s_dn;
                for (int u = b; u < units && ok; u += G) {
                    const FUnit t = f_unit(u, Nw, K, splits);
                    for (int kb = t.kb0; kb < t.kb1; ++kb) {
                        // the slot's previous GEMM stage must have its token half first
                        while (ph - pt >= kFStages) {
                            if (!issue_token(pt)) {
                                ok = false;
                                break;
                            }
                            ++pt;
                        }
                        if (!ok) break;
                        if (!mbar_wait_bounded(empty0 + 8 * slot, ephase ^ 1u, status, tmo, 44)) {
                            ok = false;
                            break;
                        }
                        const uint32_t fb = gfull0 + 8 * slot;
                        mbar_arrive_expect_tx(fb, kFWBytes);
                        tma_load_3d(smem_base + slot * kFSlot, phase == 0 ? &tm_wup : &tm_wdn, fb, kb * kRK, t.w0,
                                    t.e);
                        // once the phase's token rows exist and no earlier stage owes
                        // its half, the token half goes with the weight half (the
                        // queue below is only for the first stages of a phase)
                        const bool both = pt == ph && (phase == 0 ? gathered : hready);
                        if (both) {
                            if (cnt_sm[t.e] > 0) {
                                mbar_arrive_expect_tx(fb, kFTBytes);
                                tma_load_2d(smem_base + slot * kFSlot + kFWBytes, phase == 0 ? &tm_xg : &tm_h, fb,
                                            kb * kRK, off_sm[t.e]);
                            } else {
                                mbar_arrive(fb);  // no tokens: the MMA warp only releases the slot
                            }
                        } else {
                            const int q = ph % kFStages;
                            pend_slot[q] = slot;
                            pend_e[q] = t.e;
                            pend_kb[q] = kb;
                            pend_dn[q] = phase;
                            ++ph;
                        }
                        gpar ^= 1u << slot;
                        if (++slot == kFStages) {
                            slot = 0;
                            ephase ^= 1u;
                        }
                        if (both) continue;
                        // token halves that can go now without waiting
                        while (pt < ph && ((pend_dn[pt % kFStages] ? hready : gathered) ||
                                           ld_acquire_u32(a.sync + (pend_dn[pt % kFStages] ? SY_H : SY_GATHERED)) >=
                                               static_cast<uint32_t>(G))) {
                            if (!issue_token(pt)) {
                                ok = false;
                                break;
                            }
                            ++pt;
                        }
                    }
                }
            }
            while (ok && pt < ph) {
                if (!issue_token(pt)) {
                    ok = false;
                    break;
                }
                ++pt;
            }
            if (!ok) {
                // complete the owed arrivals so that the copies in flight can be waited for
                for (int i = pt; i < ph; ++i) mbar_arrive(gfull0 + 8 * pend_slot[i % kFStages]);
                // the last phase of every slot's barriers (a slot never used
                // passes at once: its "previous" phase counts as complete)
                for (int s2 = 0; s2 < kFStages; ++s2) {
                    wait_until(gfull0 + 8 * s2, ((gpar >> s2) & 1u) ^ 1u, tmo);
                    wait_until(rfull0 + 8 * s2, ((rpar >> s2) & 1u) ^ 1u, tmo);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int slot = 0;
            uint32_t gpar = 0, rpar = 0;
            bool ok = true, any = false;
            for (int kb = rkb0; kb < rkb1 && ok; ++kb) {
                const uint32_t par = (rpar >> slot) & 1u;
                if (!mbar_wait_bounded(rfull0 + 8 * slot, par, status, tmo, 45) ||
                    !mbar_wait_bounded(rsplit0 + 8 * slot, par, status, tmo, 46)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                mma_stage<1>(smem_base + slot * kFSlot, tmem_base + kFRouteCol, kb == rkb0);
                any = true;
                umma_commit(empty0 + 8 * slot);
                rpar ^= 1u << slot;
                if (++slot == kFStages) slot = 0;
            }
            if (ok && router_cta) umma_commit(racc);
            int local = 0;
            for (int phase = 0; phase < 2 && ok; ++phase) {
                const int units = phase == 0 ? units_up : units_dn;
                const int Nw = phase == 0 ? d_ff : d, K = phase == 0 ? d : d_ff;
                const int splits = phase == 0 ? a.s_up : a.s_dn;
                for (int u = b; u < units && ok; u += G) {
                    const FUnit t = f_unit(u, Nw, K, splits);
                    // the first stage's token half implies the routing is final
                    if (!mbar_wait_bounded(gfull0 + 8 * slot, (gpar >> slot) & 1u, status, tmo, 47)) {
                        ok = false;
                        break;
                    }
                    const int cnt = *reinterpret_cast<volatile const int32_t *>(cnt_sm + t.e);
                    const int acc = local & 1;
                    if (cnt > 0) {
                        if (!mbar_wait_bounded(tempty0 + 8 * acc, ((local >> 1) & 1) ^ 1u, status, tmo, 48)) {
                            ok = false;
                            break;
                        }
                    }
                    const int n_mma = ((cnt < kFBN ? cnt : kFBN) + 15) & ~15;
                    const uint32_t idesc = idesc_bf16_f32(128, n_mma > 0 ? n_mma : 16);
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kFBN);
                    for (int kb = t.kb0; kb < t.kb1; ++kb) {
                        if (kb > t.kb0 &&
                            !mbar_wait_bounded(gfull0 + 8 * slot, (gpar >> slot) & 1u, status, tmo, 47)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        if (cnt > 0) {
                            const uint32_t sa = smem_base + slot * kFSlot;
                            const uint64_t ad = smem_desc_sw128(sa);
                            const uint64_t bd = smem_desc_sw128(sa + kFWBytes);
#pragma unroll
                            for (int kk = 0; kk < kRK / 16; ++kk)
                                umma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb > t.kb0 || kk > 0) ? 1u : 0u);
                            any = true;
                            umma_commit(empty0 + 8 * slot);
                        } else {
                            mbar_arrive(empty0 + 8 * slot);
                        }
                        gpar ^= 1u << slot;
                        if (++slot == kFStages) slot = 0;
                    }
                    if (!ok) break;
                    if (cnt > 0) {
                        umma_commit(tfull0 + 8 * acc);
                        ++local;
                    }
                }
            }
            if (!ok && any) {
                umma_commit(drain);
                wait_until(drain, 0, tmo);
            }
        }
    } else {
        // ------------------------------------------------ warps 2-5: everything else
        const int et = threadIdx.x - 64;  // 0..127
        const int q = warp & 3;           // TMEM lane quarter
        const int row = q * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        bool ok = true;
        // 1. router piece: split W_g into the B slots, then drain the sums
        if (router_cta) {
            int slot = 0;
            uint32_t rpar = 0;
            for (int kb = rkb0; kb < rkb1; ++kb) {
                ok = __all_sync(0xffffffffu, ok);
                if (ok) ok = mbar_wait_warp(rfull0 + 8 * slot, (rpar >> slot) & 1u, status, tmo, 49);
                if (ok) {
                    split_stage<1>(smem_gen + slot * kFSlot, et);
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(rsplit0 + 8 * slot);
                rpar ^= 1u << slot;
                if (++slot == kFStages) slot = 0;
            }
            ok = __all_sync(0xffffffffu, ok);
            if (ok) ok = mbar_wait_warp(racc, 0, status, tmo, 50);
            tc_fence_after();
            if (ok) {
                float run[16];
                drain_piece<1>(tmem_base + lane_off + kFRouteCol, true, run);
                if (row < N) {
                    float *pc = a.pieces + (static_cast<int64_t>(b) * N + row) * E;
                    for (int e = 0; e < E; ++e) pc[e] = run[e];
                }
            } else if (lane == 0) {
                fail_s = 1;
            }
            tc_fence_before();
            ok = epi_arrive(a, SY_PIECES, et, &fail_s);
        }
        // 2. CTA 0: the router's finish and the slot assignment
        if (b == 0) {
            ok = epi_wait(a, SY_PIECES, static_cast<uint32_t>(a.S), et, status, 51, &fail_s);
            if (ok && et < N) {
                const int t = et;
                float run[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) run[e] = 0.0f;
                for (int e = 0; e < E; ++e) {
                    float v = a.pieces[static_cast<int64_t>(t) * E + e];
                    for (int c = 1; c < a.S; ++c) v = __fadd_rn(v, a.pieces[(static_cast<int64_t>(c) * N + t) * E + e]);
                    if (a.b_g) v = __fadd_rn(v, a.b_g[e]);
                    if (a.logits_out) a.logits_out[static_cast<int64_t>(t) * E + e] = v;
                    if (a.noise != nullptr && a.sigma != 0.0f)
                        v = __fadd_rn(v, __fmul_rn(a.sigma, a.noise[static_cast<int64_t>(t) * E + e]));
                    run[e] = v;
                }
                pick_row_regs<16>(run, E, k, pick_s + t * k, a.topk + static_cast<int64_t>(t) * k,
                                  a.gates + static_cast<int64_t>(t) * k);
            }
            epilogue_sync();
            // slots: choice j of all tokens before choice j + 1; tokens in order
            if (ok) {
                if (et < 16) sl_tot[et] = 0;
                epilogue_sync();
                if (et < N)
                    for (int j = 0; j < k; ++j) atomicAdd(&sl_tot[a.topk[et * k + j]], 1);
                epilogue_sync();
                if (et == 0) {
                    int run = 0;
                    for (int e = 0; e < E; ++e) {
                        const int c = sl_tot[e] < a.C ? sl_tot[e] : static_cast<int>(a.C);
                        a.counts[e] = c;
                        a.offsets[e] = run;
                        run += c;
                        sl_off[e] = 0;  // places handed out so far
                    }
                    a.offsets[E] = run;
                }
                epilogue_sync();
                const unsigned lt = (1u << lane) - 1u;
                for (int j = 0; j < k; ++j) {
                    const int e = et < N ? a.topk[et * k + j] : -1;
                    const unsigned same = __match_any_sync(0xffffffffu, e);
                    const int rank = __popc(same & lt);
                    if (et < 16) sl_w0[et] = 0;
                    epilogue_sync();
                    if (warp == 2 && e >= 0 && rank == 0) sl_w0[e] = __popc(same);  // tokens 0..31
                    epilogue_sync();
                    if (e >= 0) {
                        const int place = sl_off[e] + (warp == 3 ? sl_w0[e] : 0) + rank;
                        a.slot[et * k + j] = place < a.C ? place : -1;
                    }
                    epilogue_sync();
                    if (e >= 0 && rank == 0) atomicAdd(&sl_off[e], __popc(same));
                    epilogue_sync();
                }
            }
            __threadfence();
            epilogue_sync();
            if (et == 0) {
                __threadfence();
                if (ok) atomicExch(a.sync + SY_ROUTED, 1u);
                else atomicExch(a.sync + SY_ABORT, 1u);
            }
        }
        // 3. every CTA: its share of the gathered rows (pair p goes to CTA p % G)
        ok = epi_wait(a, SY_ROUTED, 1u, et, status, 52, &fail_s);
        if (ok) {
            const int chunks = d / 8;  // 16-byte pieces of a row
            for (int p = b; p < N * k; p += G) {
                const int s = a.slot[p];
                if (s < 0) continue;
                const int64_t row = static_cast<int64_t>(a.offsets[a.topk[p]]) + s;
                const uint4 *src = reinterpret_cast<const uint4 *>(a.x + static_cast<int64_t>(p / k) * d);
                uint4 *dst = reinterpret_cast<uint4 *>(a.xg + row * d);
                for (int c = et; c < chunks; c += 128) dst[c] = src[c];
            }
        }
        ok = epi_arrive(a, SY_GATHERED, et, &fail_s);
        // 4-7. the expert FFN and the combine
        int local = 0;
        for (int phase = 0; phase < 2; ++phase) {
            const int units = phase == 0 ? units_up : units_dn;
            const int Nw = phase == 0 ? d_ff : d, K = phase == 0 ? d : d_ff;
            const int splits = phase == 0 ? a.s_up : a.s_dn;
            float *parts = phase == 0 ? a.parts_up : a.parts_dn;
            const int64_t pstride = phase == 0 ? a.up_stride : a.dn_stride;
            for (int u = b; u < units && ok; u += G) {
                const FUnit t = f_unit(u, Nw, K, splits);
                const int cnt = a.counts[t.e];
                if (cnt == 0) continue;
                const int acc = local & 1;
                ok = __all_sync(0xffffffffu, ok);
                if (ok) ok = mbar_wait_warp(tfull0 + 8 * acc, (local >> 1) & 1, status, tmo, 53);
                if (!ok && lane == 0) fail_s = 1;
                tc_fence_after();
                if (ok) {
                    const int64_t rbase = a.offsets[t.e];
                    const int w = t.w0 + row;
                    const int chunks = (cnt + 31) >> 5;
                    for (int c = 0; c < chunks; ++c) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(tmem_base + lane_off + static_cast<uint32_t>(acc * kFBN + c * 32), r);
                        tmem_wait_ld();
                        if (w < Nw) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                const int tok = c * 32 + i;
                                if (tok < cnt) parts[t.split * pstride + (rbase + tok) * Nw + w] = __uint_as_float(r[i]);
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
                ++local;
            }
            ok = epi_arrive(a, phase == 0 ? SY_UP : SY_DOWN, et, &fail_s);
            if (phase == 0) {
                // 5. H = ReLU(sum of the up partials in split order), rounded to bf16
                ok = epi_wait(a, SY_UP, static_cast<uint32_t>(G), et, status, 54, &fail_s);
                if (ok) {
                    const int64_t rows = a.offsets[E];
                    const int64_t total = rows * (d_ff / 4);
                    // eight 16-byte pieces per thread in flight at a time; each piece
                    // sums the partials in split order
                    constexpr int kB = 8;
                    const int64_t step = static_cast<int64_t>(G) * 128;
                    const float4 *pu = reinterpret_cast<const float4 *>(a.parts_up);
                    for (int64_t i0 = static_cast<int64_t>(b) * 128 + et; i0 < total; i0 += kB * step) {
                        float4 v[kB];
#pragma unroll
                        for (int j = 0; j < kB; ++j) {
                            const int64_t i = i0 + j * step;
                            v[j] = i < total ? pu[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                        for (int p = 1; p < a.s_up; ++p) {
                            float4 w4[kB];
                            const float4 *pp = reinterpret_cast<const float4 *>(a.parts_up + p * a.up_stride);
#pragma unroll
                            for (int j = 0; j < kB; ++j) {
                                const int64_t i = i0 + j * step;
                                w4[j] = i < total ? pp[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                            }
#pragma unroll
                            for (int j = 0; j < kB; ++j) {
                                v[j].x += w4[j].x; v[j].y += w4[j].y; v[j].z += w4[j].z; v[j].w += w4[j].w;
                            }
                        }
#pragma unroll
                        for (int j = 0; j < kB; ++j) {
                            const int64_t i = i0 + j * step;
                            if (i < total) {
                                __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(a.H) + 2 * i;
                                o[0] = __floats2bfloat162_rn(fmaxf(v[j].x, 0.0f), fmaxf(v[j].y, 0.0f));
                                o[1] = __floats2bfloat162_rn(fmaxf(v[j].z, 0.0f), fmaxf(v[j].w, 0.0f));
                            }
                        }
                    }
                }
                ok = epi_arrive(a, SY_H, et, &fail_s);
            }
        }
        // 7. combine: token t = b, b + G, ...; the down partials summed in split
        // order, then gate-weighted in choice order
        ok = epi_wait(a, SY_DOWN, static_cast<uint32_t>(G), et, status, 55, &fail_s);
        if (ok) {
            for (int t = b; t < N; t += G) {
                for (int c8 = et; c8 < d / 8; c8 += 128) {
                    const int c = c8 * 8;
                    float acc8[8];
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc8[v] = 0.0f;
                    for (int j = 0; j < k; ++j) {
                        const int s = a.slot[t * k + j];
                        if (s < 0) continue;
                        const int64_t r = static_cast<int64_t>(a.offsets[a.topk[t * k + j]]) + s;
                        float o[8];
                        const float4 *p0 = reinterpret_cast<const float4 *>(a.parts_dn + r * d + c);
                        float4 lo = p0[0], hi = p0[1];
                        o[0] = lo.x; o[1] = lo.y; o[2] = lo.z; o[3] = lo.w;
                        o[4] = hi.x; o[5] = hi.y; o[6] = hi.z; o[7] = hi.w;
                        for (int p = 1; p < a.s_dn; ++p) {
                            const float4 *pp = reinterpret_cast<const float4 *>(a.parts_dn + p * a.dn_stride + r * d + c);
                            lo = pp[0];
                            hi = pp[1];
                            o[0] += lo.x; o[1] += lo.y; o[2] += lo.z; o[3] += lo.w;
                            o[4] += hi.x; o[5] += hi.y; o[6] += hi.z; o[7] += hi.w;
                        }
                        const float gj = a.gates[t * k + j];
#pragma unroll
                        for (int v = 0; v < 8; ++v) acc8[v] = fmaf(gj, o[v], acc8[v]);
                    }
                    uint4 packed;
                    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&packed);
#pragma unroll
                    for (int v = 0; v < 4; ++v) h[v] = __floats2bfloat162_rn(acc8[2 * v], acc8[2 * v + 1]);
                    *reinterpret_cast<uint4 *>(a.y + static_cast<int64_t>(t) * d + c) = packed;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) publish_status(a.status, cta_status);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kFTmemCols);
    }
}

}  // namespace

bool decode_fused_eligible(const void *x, const float *W_g, int64_t N, int d, int E, int d_ff, int k, int64_t rows,
                           int num_sms) {
    return N >= 1 && N <= kFBN && d % 8 == 0 && d_ff % 8 == 0 && E >= 1 && E <= 16 && k >= 1 && k <= kFMaxK &&
           k <= E && rows <= 256 && route_tc_eligible(x, W_g, N, d, E, k) && route_k_splits(d) < num_sms &&
           num_sms >= 2;
}

size_t decode_fused_scratch_bytes(int64_t N, int d, int E) {
    return align_up(sizeof(uint32_t) * SY_WORDS, 256) +
           align_up(sizeof(float) * static_cast<size_t>(route_k_splits(d)) * N * E, 256);
}

cudaError_t launch_decode_fused(const void *x, const float *W_g, const float *b_g, const float *noise, float sigma,
                                int64_t N, int d, int E, int d_ff, int k, int64_t C, const void *W_up,
                                const void *W_down, void *y, float *logits_out, int32_t *topk, float *gates,
                                int32_t *slot, int32_t *counts, int32_t *offsets, void *xg, int64_t rows, void *H,
                                float *parts_dn, float *parts_up, int s_up, int s_dn, void *scratch,
                                uint32_t *status, uint64_t timeout_ns, int num_sms, cudaStream_t s) {
    CUtensorMap tm_x, tm_wg, tm_wup, tm_wdn, tm_xg, tm_h;
    if (!make_tmap_bf16_2d(&tm_x, x, N, d, kRM)) return cudaErrorInvalidValue;
    if (!make_tmap_f32_2d(&tm_wg, W_g, E, d, 16, kRK)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_3d(&tm_wup, W_up, E, d_ff, d, 128)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_3d(&tm_wdn, W_down, E, d, d_ff, 128)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tm_xg, xg, rows, d, kFBN)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tm_h, H, rows, d_ff, kFBN)) return cudaErrorInvalidValue;
    uint8_t *sc = static_cast<uint8_t *>(scratch);
    uint32_t *sync = reinterpret_cast<uint32_t *>(sc);
    float *pieces = reinterpret_cast<float *>(sc + align_up(sizeof(uint32_t) * SY_WORDS, 256));
    cudaError_t e = cudaMemsetAsync(sync, 0, sizeof(uint32_t) * SY_WORDS, s);
    if (e != cudaSuccess) return e;
    FusedArgs a{static_cast<const __nv_bfloat16 *>(x), b_g, noise, sigma, static_cast<int>(N), d, E, k, d_ff, C,
                route_k_splits(d), s_up, s_dn, logits_out, topk, slot, counts, offsets, gates,
                static_cast<__nv_bfloat16 *>(xg), static_cast<__nv_bfloat16 *>(H), static_cast<__nv_bfloat16 *>(y),
                parts_up, parts_dn, rows * static_cast<int64_t>(d_ff), rows * static_cast<int64_t>(d), pieces, sync,
                status, timeout_ns};
    constexpr size_t smem = static_cast<size_t>(kFStages) * kFSlot + 1024;
    e = cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(num_sms));
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid-wide waits end
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_fused_kernel, tm_x, tm_wg, tm_wup, tm_wdn, tm_xg, tm_h, a);
}

}  // namespace moe
