// Router building blocks shared by the router kernels (route_tc.cu) and the
// fused small-batch layer (decode_fused.cu): the exact three-way bf16 split
// of the fp32 router weights, the stage layout and MMAs of one K block, the
// K pieces, the drain of a piece, and KeepTopK + softmax of one token.  Both
// users run this same code, so a token's logits, picks and gates come out bit
// for bit the same whichever kernel routed it.
//
// Accumulators of one piece: 3 * E_pad fp32 columns of tensor memory, column
// c summing the products with row c of B = [w_hi; w_mid; w_lo] (one MMA of
// N = 3 * E_pad per 16-wide K step: each step reads the x tile from shared
// memory once).  The piece's value is (hi-sum + mid-sum) + lo-sum.
//
// "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター" STEP 2 and 4-6;
// "nanoMoEの深層解剖" slides 11-13.
#pragma once

#include "common.cuh"
#include "tmap.h"

namespace moe {
namespace rt {
namespace {

constexpr int kRM = 128;                           // tokens per tile (MMA M)
constexpr int kRK = kTmapBoxK;                     // K elements per stage
constexpr uint32_t kXTileBytes = kRM * kRK * 2;    // 16 KB of bf16 tokens per stage

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

template <int UPT>
__host__ __device__ constexpr int route_nb() {  // rows of B: [w_hi; w_mid; w_lo]
    return 3 * 16 * UPT;
}
template <int UPT>
__host__ __device__ constexpr int route_acc_cols() {  // accumulator columns of one piece
    return 3 * 16 * UPT;
}

// One ring stage: the x tile (bf16, 128-byte swizzle), the B slot (3 * E_pad
// bf16 rows, 128-byte swizzle) and, for the in-kernel split, the fp32 W_g tile
// the B slot is split from (E_pad rows of 64, unswizzled, zero past E).
template <int UPT>
__host__ __device__ constexpr uint32_t route_b_bytes() {
    return static_cast<uint32_t>(route_nb<UPT>()) * kRK * 2u;
}
template <int UPT, bool PRE>
__host__ __device__ constexpr uint32_t route_wtile_bytes() {
    return PRE ? 0u : 16u * UPT * kRK * 4u;
}
template <int UPT, bool PRE>
__host__ __device__ constexpr uint32_t route_stage_bytes() {
    return kXTileBytes + route_b_bytes<UPT>() + route_wtile_bytes<UPT, PRE>();
}
// Rows of B per TMA box when pre-split (a box holds at most 256 rows).
template <int UPT>
__host__ __device__ constexpr int route_b_box_rows() {
    return route_nb<UPT>() <= 256 ? route_nb<UPT>() : route_nb<UPT>() / 2;
}

// TMA loads of one stage: the x tile of rows row0.. and K block kb, and B
// (pre-split) or the fp32 W_g tile (in-kernel split), all on barrier `bar`.
template <int UPT, bool PRE>
__device__ __forceinline__ void load_stage(uint32_t st, const CUtensorMap *tm_x, const CUtensorMap *tm_w,
                                           uint32_t bar, int kb, int row0, int tile_rows) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(tile_rows) * kRK * 2u +
                                   (PRE ? route_b_bytes<UPT>() : route_wtile_bytes<UPT, PRE>()));
    tma_load_2d(st, tm_x, bar, kb * kRK, row0);
    if constexpr (PRE) {
        constexpr int box = route_b_box_rows<UPT>();
#pragma unroll
        for (int r = 0; r < route_nb<UPT>(); r += box)
            tma_load_2d(st + kXTileBytes + static_cast<uint32_t>(r) * 128u, tm_w, bar, kb * kRK, r);
    } else {
        tma_load_2d(st + kXTileBytes + route_b_bytes<UPT>(), tm_w, bar, kb * kRK, 0);
    }
}

// In-kernel split of the fp32 W_g tile of one stage into its B slot.  Thread
// et (0..127) of the splitting warps owns units et + 128 i: expert row u / 8,
// 8-column chunk u % 8.
template <int UPT>
__device__ __forceinline__ void split_stage(uint8_t *stage_gen, int et) {
    constexpr int E_PAD = 16 * UPT;
    const float *wt = reinterpret_cast<const float *>(stage_gen + kXTileBytes + route_b_bytes<UPT>());
    uint8_t *bbase = stage_gen + kXTileBytes;
#pragma unroll
    for (int i = 0; i < UPT; ++i) {
        const int u = et + i * 128;
        const int e = u >> 3, c = u & 7;
        const float4 a = *reinterpret_cast<const float4 *>(wt + e * kRK + c * 8);
        const float4 b = *reinterpret_cast<const float4 *>(wt + e * kRK + c * 8 + 4);
        uint4 hi, mid, lo;
        split3(a.x, a.y, hi.x, mid.x, lo.x);
        split3(a.z, a.w, hi.y, mid.y, lo.y);
        split3(b.x, b.y, hi.z, mid.z, lo.z);
        split3(b.z, b.w, hi.w, mid.w, lo.w);
        *reinterpret_cast<uint4 *>(bbase + sw128_offset(e, c)) = hi;
        *reinterpret_cast<uint4 *>(bbase + sw128_offset(E_PAD + e, c)) = mid;
        *reinterpret_cast<uint4 *>(bbase + sw128_offset(2 * E_PAD + e, c)) = lo;
    }
}

__host__ __device__ constexpr uint32_t tmem_alloc_cols(int cols) {  // a power of two, at least 32
    return cols <= 32 ? 32 : cols <= 64 ? 64 : cols <= 128 ? 128 : cols <= 256 ? 256 : 512;
}
template <int UPT>
__host__ __device__ constexpr uint32_t route_tmem_cols() {  // clustered: one buffer
    return tmem_alloc_cols(route_acc_cols<UPT>());
}
// Persistent form: piece buffers in tensor memory (up to 4), so the MMAs run
// ahead of the drains by up to that many pieces.
template <int UPT>
__host__ __device__ constexpr int routep_nbuf() {
    return 512 / route_acc_cols<UPT>() < 4 ? 512 / route_acc_cols<UPT>() : 4;
}
template <int UPT>
__host__ __device__ constexpr uint32_t routep_tmem_cols() {
    return tmem_alloc_cols(routep_nbuf<UPT>() * route_acc_cols<UPT>());
}

// Which K blocks piece c of S sums: [c*kb/S, (c+1)*kb/S).
__host__ __device__ inline int route_kb_begin(int c, int S, int kb_total) {
    return static_cast<int>(static_cast<int64_t>(c) * kb_total / S);
}

// Pieces of K: at least 8 blocks (512 columns) each, at most 8.  S depends
// on d only.
__host__ __device__ inline int route_k_splits(int d) {
    const int kb_total = (d + kRK - 1) / kRK;
    const int s = (kb_total + 7) / 8;
    return s < 1 ? 1 : (s > 8 ? 8 : s);
}

// MMAs of one stage into the piece accumulator at d_tmem (N = 3 * E_pad,
// issued in chunks of at most 256 columns); acc0 = true starts the piece.
template <int UPT>
__device__ __forceinline__ void mma_stage(uint32_t st, uint32_t d_tmem, bool acc0) {
    constexpr int NB = route_nb<UPT>();
    const uint64_t ad = smem_desc_sw128(st);
#pragma unroll
    for (int kk = 0; kk < kRK / 16; ++kk) {
#pragma unroll
        for (int n0 = 0; n0 < NB; n0 += 256) {
            const int nn = (NB - n0) < 256 ? (NB - n0) : 256;
            const uint64_t bd = smem_desc_sw128(st + kXTileBytes + static_cast<uint32_t>(n0) * 128u);
            // +32 bytes along K inside the swizzled row = +2 in the address field
            umma_bf16(d_tmem + static_cast<uint32_t>(n0), ad + 2 * kk, bd + 2 * kk, idesc_bf16_f32(kRM, nn),
                      (!acc0 || kk > 0) ? 1u : 0u);
        }
    }
}

// The piece sums of experts [16 ch, 16 ch + 16) for this thread's token row:
// (hi + mid) + lo, from the piece accumulator at taddr.
template <int UPT>
__device__ __forceinline__ void piece_chunk(uint32_t taddr, int ch, float (&p)[16]) {
    constexpr int EP = 16 * UPT;
    uint32_t h[16], m[16], l[16];
    tmem_ld_32x32b_x16(taddr + ch * 16, h);
    tmem_ld_32x32b_x16(taddr + EP + ch * 16, m);
    tmem_ld_32x32b_x16(taddr + 2 * EP + ch * 16, l);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i)
        p[i] = __fadd_rn(__fadd_rn(__uint_as_float(h[i]), __uint_as_float(m[i])), __uint_as_float(l[i]));
}

// Sum of one piece for this thread's token row into run: the piece sum
// (first piece) or run + piece sum, for the experts of chunks [ch0, ch0 + NCH).
template <int UPT, int NCH = UPT>
__device__ __forceinline__ void drain_piece(uint32_t taddr, bool first, float (&run)[16 * NCH], int ch0 = 0) {
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
        float p[16];
        piece_chunk<UPT>(taddr, ch0 + ch, p);
#pragma unroll
        for (int i = 0; i < 16; ++i) run[ch * 16 + i] = first ? p[i] : __fadd_rn(run[ch * 16 + i], p[i]);
    }
}

// KeepTopK and softmax of one token (one thread): k rounds, each taking the
// best score ranked after the previous pick (score descending, lower expert
// index first on ties); then the softmax over the kept scores.  pv_s: this
// thread's k floats of scratch.  Scores in shared memory (sr[0..E)).
__device__ __forceinline__ void pick_row_smem(const float *sr, int E, int k, float *pv_s, int32_t *ti, float *gt) {
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
        pv_s[j] = bv;
        pv = bv;
        pe = be;
    }
    const float mx = pv_s[0];
    float sum = 0.0f;
    for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, expf(__fsub_rn(pv_s[j], mx)));
    for (int j = 0; j < k; ++j) gt[j] = __fdiv_rn(expf(__fsub_rn(pv_s[j], mx)), sum);
}

// The same for scores held in registers (s[0..E), E <= E_PAD; s is consumed).
// Each score becomes a 32-bit word whose unsigned order is the float order
// (-0 taken as +0, so equal floats give equal words; every finite score maps
// above 0).  A round takes, among the experts not picked yet, the largest
// word and the lowest index among equal words: eight running (word, index)
// pairs over e = i, i + 8, ... (a later e replaces the pair only when its
// word is strictly larger), folded with ties going to the lower index.
// Picked experts are bits of a mask.
__device__ __forceinline__ uint32_t ordered_bits(float v) {
    const uint32_t b = __float_as_uint(v == 0.0f ? 0.0f : v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float from_ordered_bits(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// Softmax over the k kept scores in pick order (the first is the largest).
__device__ __forceinline__ void softmax_kept(const float *pv_s, int k, float *gt) {
    const float mx = pv_s[0];
    float sum = 0.0f;
    for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, expf(__fsub_rn(pv_s[j], mx)));
    for (int j = 0; j < k; ++j) gt[j] = __fdiv_rn(expf(__fsub_rn(pv_s[j], mx)), sum);
}

template <int E_PAD>
__device__ __forceinline__ void pick_row_regs(float (&s)[E_PAD], int E, int k, float *pv_s, int32_t *ti,
                                              float *gt) {
    constexpr int W = (E_PAD + 31) / 32;
    uint32_t u[E_PAD];
#pragma unroll
    for (int e = 0; e < E_PAD; ++e) u[e] = e < E ? ordered_bits(s[e]) : 0u;  // 0: never picked
    uint32_t picked[W];
#pragma unroll
    for (int w = 0; w < W; ++w) picked[w] = 0u;
    for (int j = 0; j < k; ++j) {
        uint32_t bu[8];
        int be[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            bu[i] = 0u;
            be[i] = E_PAD;
        }
#pragma unroll
        for (int e = 0; e < E_PAD; ++e) {
            const bool taken = (picked[e >> 5] >> (e & 31)) & 1u;
            if (!taken && u[e] > bu[e & 7]) {
                bu[e & 7] = u[e];
                be[e & 7] = e;
            }
        }
        uint32_t best = bu[0];
        int arg = be[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
            if (bu[i] > best || (bu[i] == best && be[i] < arg)) {
                best = bu[i];
                arg = be[i];
            }
        }
        ti[j] = arg;
        pv_s[j] = from_ordered_bits(best);
#pragma unroll
        for (int w = 0; w < W; ++w)
            if ((arg >> 5) == w) picked[w] |= 1u << (arg & 31);
    }
    softmax_kept(pv_s, k, gt);
}

// KeepTopK over one part of a token's experts, [e0, e0 + H) of which those
// below E count: k rounds as above, writing each round's word and expert index
// (word 0 once the part has no expert left).  The two parts' lists, each in
// pick order, merge into the token's picks (merge_picks).
template <int H>
__device__ __forceinline__ void pick_part_regs(float (&s)[H], int e0, int E, int k, uint32_t *wo, int32_t *io) {
    constexpr int W = (H + 31) / 32;
    uint32_t u[H];
#pragma unroll
    for (int e = 0; e < H; ++e) u[e] = e0 + e < E ? ordered_bits(s[e]) : 0u;
    uint32_t picked[W];
#pragma unroll
    for (int w = 0; w < W; ++w) picked[w] = 0u;
    for (int j = 0; j < k; ++j) {
        uint32_t bu[8];
        int be[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            bu[i] = 0u;
            be[i] = H;
        }
#pragma unroll
        for (int e = 0; e < H; ++e) {
            const bool taken = (picked[e >> 5] >> (e & 31)) & 1u;
            if (!taken && u[e] > bu[e & 7]) {
                bu[e & 7] = u[e];
                be[e & 7] = e;
            }
        }
        uint32_t best = bu[0];
        int arg = be[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
            if (bu[i] > best || (bu[i] == best && be[i] < arg)) {
                best = bu[i];
                arg = be[i];
            }
        }
        wo[j] = best;
        io[j] = e0 + arg;
#pragma unroll
        for (int w = 0; w < W; ++w)
            if ((arg >> 5) == w) picked[w] |= 1u << (arg & 31);
    }
}

// The token's k picks from the pick lists of its lower experts (a) and its
// upper experts (b), each in pick order: a merge of the two orders, equal
// words going to a (its experts have the lower indices).  Scores to pv_s,
// experts to ti.
__device__ __forceinline__ void merge_picks(const uint32_t *aw, const int32_t *ai, const uint32_t *bw,
                                            const int32_t *bi, int k, float *pv_s, int32_t *ti) {
    int i = 0, j = 0;
    for (int n = 0; n < k; ++n) {
        const uint32_t wa = i < k ? aw[i] : 0u, wb = j < k ? bw[j] : 0u;
        if (wa >= wb) {
            ti[n] = ai[i];
            pv_s[n] = from_ordered_bits(wa);
            ++i;
        } else {
            ti[n] = bi[j];
            pv_s[n] = from_ordered_bits(wb);
            ++j;
        }
    }
}

}  // namespace
}  // namespace rt
}  // namespace moe
