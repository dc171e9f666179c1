// attend.cuh -- the streaming part of the decode kernel: split-K
// pruned-channel attention over the INT2 paged cache ("Throughput on SGLang":
// pruning removes 40 % of key channels from reads, quantization cuts storage
// to 2 bits per value) -- unit bookkeeping, the producer warp, and the
// per-page consumer steps -- and k_merge, the merge of context-parallel
// records.
//
// Work split: the cache is a sequence of units (pages of one run; a run is a
// (sequence, chunk of <= 8 kv heads)).  CTA c of C owns units
// [floor(c*U/C), floor((c+1)*U/C)): every CTA streams the same number of pages
// whatever the length mix.  A producer warp brings whole units in with 1-D bulk
// async copies (one copy = 16 tokens x up to 8 kv heads, contiguous) into a
// ring of shared-memory stages of 16 (page, kv head) blocks guarded by
// mbarriers.  Consumer warps each own one kv head and take two or four pages
// of it per stage, processed together (independent instruction streams).
//
// Per consumer warp and page (16 tokens x G query heads), with
// qs = q' * log2(e)/sqrt(d) on the kept channels:
//   QK   D_g[t, n] = sum_{c in g} code[t, c] * Q[c, n]    (m16n8k32 u8 x s8, per group)
//        n = (head, piece): qs ~= sigma_g (Q1 + Q2/256) in two int8 pieces placed
//        in the columns a GQA group of 4 leaves free, sigma_g = sigma_h 2^-e_g
//        (15-16 bits relative to the group's largest |qs|); one AND per 4 codes
//        forms the u8 operand (code * 4^g);
//        s[t, h] = sigma_h * sum_g scale[t, g] * p_g * (D_g[t,(h,1)] + D_g[t,(h,2)]/256)
//                + sum_g min[t, g] * Qsum[g, h]   (one extra m16n8k16; the high and
//                                                  low fp16 parts of Qsum in separate rows)
//                + qs_0[h] * k0[t]                (BF16 channel 0, fp32)
//        with p_g = 2^-e_g / 4^g.  256 D1 + D2 is exact in int32 (below 2^28);
//        it becomes fp32 with one rounding, and scale[t, g] * p_g / 256 is
//        exact (p_g a power of two), so one FFMA adds
//        scale * p_g (D1 + D2/256) with the roundings of the definition.
//   online softmax in base 2 (running max per head, exact rescale on growth)
//   PV   O^T[c, h] += sum_t code_v[t, c] * (p~[t, h] * vscale[t, g(c)])
//        with p~ = fp16(p); one extra m16n8k16 gives sum_t p~ * vmin[t, g] and
//        l = sum_t p~ (a row of ones), so numerator and denominator see the
//        same rounded weights.
// Value codes become exact fp16 operands with one AND per register: with
// head_dim 128 as subnormals (code * 4^P * 2^-24, P the field position, the
// power of two removed when a run is finished), with head_dim 64 through a
// magic exponent and one HSUB2.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace dqk {

// CTA shape of the decode kernel's streaming loop: consumer warps, each owning
// one kv head of a chunk and taking attend_pages_per_warp pages of it per
// stage (processed as independent instruction streams), plus one producer
// warp.  Twelve consumer warps taking four pages each where the per-warp state
// allows (G <= 4; thirteen warps keep 128 registers a thread, since the
// register file is split between the four schedulers), eight taking two for
// G = 8, whose two query-head tiles double that state.
__host__ __device__ constexpr int attend_warps(int G) { return G > 4 ? 8 : 12; }
__host__ __device__ constexpr int attend_pages_per_warp(int G) { return G > 4 ? 2 : 4; }
__host__ __device__ constexpr int attend_stage_blocks(int G) { return attend_pages_per_warp(G) * attend_warps(G); }
__host__ __device__ constexpr int attend_threads(int G) { return 32 * (attend_warps(G) + 1); }
constexpr int kMaxStages = 8;                               // ring depth cap
constexpr uint64_t kWaitLimitNs = 1000000000ull;            // 1 s: a stuck pipeline reports DQK_ERR_TIMEOUT

struct AttendParams {
    const uint8_t *pool;
    long long num_pages;
    const int *seq_lens;
    const int *page_table;
    const uint2 *qf;
    const float *qk;
    const uint32_t *qm;
    const float *q0;
    float *part;
    int batch, hq, hkv, hc, pps, pw, nchunks, max_pages, bb, v_ch0, stages, num_ctas;
};

// ---------------------------------------------------------------------------
// unit bookkeeping (runs r = b*nchunks + chunk, ceil(L_b/16) pages each)
// ---------------------------------------------------------------------------
__device__ __forceinline__ int run_pages(const int *seq_lens, int nchunks, int r) {
    const int L = seq_lens[r / nchunks];
    return L > 0 ? (L + kPage - 1) / kPage : 0;
}

__device__ __forceinline__ long long warp_total_units(const int *seq_lens, int nchunks, int R, int lane) {
    long long s = 0;
    for (int r = lane; r < R; r += 32) s += run_pages(seq_lens, nchunks, r);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// The run holding unit u and the unit where it starts (warp-uniform result).
// Returns r = R when u is past the last unit.
__device__ __forceinline__ void warp_locate(const int *seq_lens, int nchunks, int R, long long u, int lane,
                                            int &r_out, long long &start_out) {
    long long base = 0;
    for (int r0 = 0; r0 < R; r0 += 32) {
        const int r = r0 + lane;
        const long long np = r < R ? run_pages(seq_lens, nchunks, r) : 0;
        long long incl = np;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const long long excl = incl - np;
        const bool hit = np > 0 && base + excl <= u && u < base + incl;
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            r_out = r0 + src;
            start_out = base + __shfl_sync(0xffffffffu, excl, src);
            return;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    r_out = R;
    start_out = base;
}

// CTA owning unit u when U units are split over C CTAs.
__host__ __device__ __forceinline__ long long cta_of_unit(long long u, long long U, long long C) {
    return ((u + 1) * C - 1) / U;
}

// The CTA's unit range [u0, u1) out of U units, the run r holding u0 and the
// unit ur where that run starts (r = R past the last unit).  One warp, one
// pass over the run lengths when there are at most 32 runs.
struct CtaUnits {
    int U, u0, u1, r, ur;
};

__device__ __forceinline__ CtaUnits cta_units(const int *seq_lens, int nchunks, int R, int cta, int num_ctas,
                                              int lane) {
    CtaUnits cu;
    if (R <= 32) {
        const int np = lane < R ? run_pages(seq_lens, nchunks, lane) : 0;
        int incl = np;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        cu.U = __shfl_sync(0xffffffffu, incl, 31);
        cu.u0 = (int)((long long)cta * cu.U / num_ctas);
        cu.u1 = (int)(((long long)cta + 1) * cu.U / num_ctas);
        const unsigned m = __ballot_sync(0xffffffffu, np > 0 && incl - np <= cu.u0 && cu.u0 < incl);
        cu.r = m ? __ffs(m) - 1 : R;
        cu.ur = m ? __shfl_sync(0xffffffffu, incl - np, cu.r) : cu.U;
    } else {
        cu.U = (int)warp_total_units(seq_lens, nchunks, R, lane);
        cu.u0 = (int)((long long)cta * cu.U / num_ctas);
        cu.u1 = (int)(((long long)cta + 1) * cu.U / num_ctas);
        long long urll;
        warp_locate(seq_lens, nchunks, R, cu.u0, lane, cu.r, urll);
        cu.ur = (int)urll;
    }
    return cu;
}

// Partial record of (slot = CTA + run, warp pair index pi, kv head jl, query head hh):
// kRecHead floats (m, l and two unused) then o[D], so o starts 16-byte aligned.
constexpr int kRecHead = 4;
__host__ __device__ constexpr int rec_stride(int D) { return kRecHead + D; }
__host__ __device__ __forceinline__ size_t record_index(int slot, int pi, int jl, int hh, int pw, int hc, int G) {
    return (((size_t)slot * pw + pi) * hc + jl) * G + hh;
}

// ---------------------------------------------------------------------------
// the attend kernel
// ---------------------------------------------------------------------------
template <int D, int G>
struct AttendTile {
    static constexpr int NG = D / 32;
    static constexpr int NT = G > 4 ? 2 : 1;   // n-tiles of 4 heads
    static constexpr int NM = D / 16;          // m-tiles of the PV product
};

// Factor that turns the PV accumulator of m-tile m into value units: 2^(24 - 2P)
// for the subnormal operands of the NG = 4 layout, 1 otherwise.
template <int NG>
__device__ __forceinline__ float vfield_scale(int m) {
    if constexpr (NG == 4) return __int_as_float((127 + 24 - 2 * (m <= 4 ? m : m - 5)) << 23);
    else return 1.0f;
}

// Online-softmax state of one consumer warp for one (run, kv head).
template <int D, int G>
struct WarpState {
    using T = AttendTile<D, G>;
    static constexpr bool kRegFrags = T::NT == 1;   // score fragments in registers (else per-warp shared memory)
    uint2 qb[kRegFrags ? T::NG : 1];                // score B fragments of group g
    float kq[kRegFrags ? T::NG : 1];                // p_g / 256 of group g
    float sgh[T::NT];              // sigma_h of this thread's head
    uint32_t qmin[T::NT];          // min-term B fragment
    float q0v[T::NT];              // scaled q'_0 of this thread's head
    float m_run[T::NT];            // running max (log2 units) of this thread's head
    float oacc[T::NT][T::NM][4];   // PV accumulators (columns 2*tig hold head tig)
    float macc[T::NT][4];          // rows: group min terms, softmax denominator, channel 0
};

// Per-lane byte offsets into a block, fixed for the kernel.
struct LaneOffsets {
    uint32_t lane16;   // lane * 16: K/V code words
    uint32_t gid8;     // (lane/4) * 8: K scales of token gid (token gid+8 at +64)
    uint32_t kmin;     // K min pair of token gid for this lane's column pair
    uint32_t gid4;     // (lane/4) * 4: K channel 0 of tokens gid, gid+8
    uint32_t tig16;    // (lane%4) * 16: V scale pairs of tokens 2tig.. (+64: 2tig+8..)
    uint32_t vmin;     // V min pair of row min(gid, NG-1), tokens 2tig, 2tig+1
    int srcA;          // lane holding p of (token 2tig, head gid/2); +4: token 2tig+1
    uint32_t sq;       // shared address of this lane's QK B fragments: [NT][NG][32 lanes] uint2
    uint32_t sk;       // shared address of this thread's head constants: [NT][NG][4 heads] 16-byte slots (p_g / 256)
    uint32_t ones_lane, vmin_mask;
};

// A page is consumed in three steps: qk_scores (scores of its 16 tokens for
// the warp's G query heads), max_update (the lazy running max) and pv_accum
// (softmax weights and the value accumulation).  NB (page, kv head) blocks at
// shared addresses sb[], same run; MASKED (NB == 1 only): only the first nv
// tokens are valid.
template <int D, int G, int NS, int NB, bool MASKED>
__device__ __forceinline__ void qk_scores(const uint32_t (&sb)[NB], int nv, const WarpState<D, G> &st, int lane,
                                          const LaneOffsets &o, float (&s0)[NB][AttendTile<D, G>::NT],
                                          float (&s1)[NB][AttendTile<D, G>::NT]) {
    using T = AttendTile<D, G>;
    constexpr int NG = T::NG, NT = T::NT;
    constexpr Layout Ly = make_layout(D, 0, NS);   // section offsets do not depend on v_ch0 (V0 is last)
    static_assert(NB == 1 || !MASKED, "masked blocks are processed alone");
    const int gid = lane >> 2;

    constexpr int KS = NS == 1 ? 1 : NG / 2;   // words of key scales per token
    uint32_t kw[NB][NG], ks0[NB][KS], ks1[NB][KS], km0[NB], km1[NB];
    float k0a[NB], k0b[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        if constexpr (NG == 4) {
            const uint4 v = ld_s128(sb[b] + o.lane16 + Ly.kc);
            kw[b][0] = v.x; kw[b][1] = v.y; kw[b][2] = v.z; kw[b][3] = v.w;
        } else {
            const uint2 v = ld_s64(sb[b] + (o.lane16 >> 1) + Ly.kc);
            kw[b][0] = v.x; kw[b][1] = v.y;
        }
        if constexpr (NS == 1) {
            // one scale and one min per token: tokens gid and gid + 8
            const uint32_t a = sb[b] + (o.gid4 >> 1);
            ks0[b][0] = ld_s16(a + Ly.ks);
            ks1[b][0] = ld_s16(a + Ly.ks + 16);
            const uint32_t m0 = ld_s16(a + Ly.km), m1 = ld_s16(a + Ly.km + 16);
            km0[b] = m0 | (m0 << 16);          // the same min against every group's Qsum
            km1[b] = m1 | (m1 << 16);
        } else {
            if constexpr (NG == 4) {
                const uint32_t a = sb[b] + o.gid8;
                const uint2 x = ld_s64(a + Ly.ks), y = ld_s64(a + Ly.ks + 64);
                ks0[b][0] = x.x; ks0[b][1] = x.y; ks1[b][0] = y.x; ks1[b][1] = y.y;
            } else {
                const uint32_t a = sb[b] + (o.gid8 >> 1);
                ks0[b][0] = ld_s32(a + Ly.ks);
                ks1[b][0] = ld_s32(a + Ly.ks + 32);
            }
            const uint32_t akm = sb[b] + o.kmin;
            // A columns k and NG + k both hold group k's min (lanes tig >= NG/2
            // repeat the pairs of the lanes below); the B operand holds the high
            // and the low fp16 part of Qsum there, so one tile sums both
            km0[b] = ld_s32(akm + Ly.km);
            km1[b] = ld_s32(akm + Ly.km + 16 * NG);
        }
        const uint32_t k0w = ld_s32(sb[b] + o.gid4 + Ly.k0);
        k0a[b] = __uint_as_float(k0w << 16);
        k0b[b] = __uint_as_float(k0w & 0xffff0000u);
    }
    // acc.x: token gid, acc.y: token gid + 8 (one packed instruction for both)
    float2 acc[NB][NT];
    float cmin[NB][NT][4];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            acc[b][nt] = make_float2(0.0f, 0.0f);
            cmin[b][nt][0] = cmin[b][nt][1] = cmin[b][nt][2] = cmin[b][nt][3] = 0.0f;
            mma_f16(cmin[b][nt], km0[b], km1[b], 0u, 0u, st.qmin[nt], 0u);
        }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const uint32_t msk = 0x03030303u << (2 * g);   // group g's field in every byte: code * 4^g
        uint2 qb[NT];
        float kq[NT];
        if constexpr (WarpState<D, G>::kRegFrags) {
            qb[0] = st.qb[g];
            kq[0] = st.kq[g];
        } else {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                qb[nt] = ld_s64(o.sq + (nt * NG + g) * 256);
                kq[nt] = __uint_as_float(ld_s32(o.sk + (nt * NG + g) * 64));
            }
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            uint32_t A0, A1, A2, A3;
            if constexpr (NG == 4) {
                A0 = kw[b][0] & msk; A1 = kw[b][1] & msk; A2 = kw[b][2] & msk; A3 = kw[b][3] & msk;
            } else {
                A0 = kw[b][0] & msk; A1 = kw[b][1] & msk;
                A2 = (kw[b][0] >> 4) & msk; A3 = (kw[b][1] >> 4) & msk;
            }
            // key scales of tokens gid and gid + 8
            float sa, sbv;
            if constexpr (NS == 1) {
                sa = f16lo_to_f32(ks0[b][0]);
                sbv = f16lo_to_f32(ks1[b][0]);
            } else {
                sa = (g & 1) ? f16hi_to_f32(ks0[b][g >> 1]) : f16lo_to_f32(ks0[b][g >> 1]);
                sbv = (g & 1) ? f16hi_to_f32(ks1[b][g >> 1]) : f16lo_to_f32(ks1[b][g >> 1]);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                int dg[4] = {0, 0, 0, 0};
                mma_u8s8_acc(dg, A0, A1, A2, A3, qb[nt].x, qb[nt].y);
                // rows gid, gid + 8: 256 D1 + D2 (exact), one rounding to fp32
                const float2 y = make_float2((float)(dg[0] * 256 + dg[1]), (float)(dg[2] * 256 + dg[3]));
                acc[b][nt] = fma2(mul2(make_float2(sa, sbv), make_float2(kq[nt], kq[nt])), y, acc[b][nt]);
            }
        }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float2 t = fma2(make_float2(st.q0v[nt], st.q0v[nt]), make_float2(k0a[b], k0b[b]),
                                  make_float2(cmin[b][nt][0], cmin[b][nt][2]));
            const float2 sv = fma2(make_float2(st.sgh[nt], st.sgh[nt]), acc[b][nt], t);
            s0[b][nt] = sv.x;
            s1[b][nt] = sv.y;
            if constexpr (MASKED) {
                if (gid >= nv) s0[b][nt] = -INFINITY;
                if (gid + 8 >= nv) s1[b][nt] = -INFINITY;
            }
        }
}

// The running max only moves when a score exceeds it (rare after the first
// pages): then take the exact max over these pages and rescale.
template <int D, int G, int NB>
__device__ __forceinline__ void max_update(WarpState<D, G> &st, const float (&s0)[NB][AttendTile<D, G>::NT],
                                           const float (&s1)[NB][AttendTile<D, G>::NT]) {
    using T = AttendTile<D, G>;
    constexpr int NT = T::NT;
    float mxs[NT];
    bool grow = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float mx = fmaxf(s0[0][nt], s1[0][nt]);
#pragma unroll
        for (int b = 1; b < NB; ++b) mx = fmaxf(mx, fmaxf(s0[b][nt], s1[b][nt]));
        mxs[nt] = mx;
        grow |= mx > st.m_run[nt];
    }
    if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float mx = mxs[nt];
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mnew = fmaxf(st.m_run[nt], mx);
            const float alpha = fast_exp2(st.m_run[nt] - mnew);   // 0 when the old max is -inf
#pragma unroll
            for (int m = 0; m < T::NM; ++m) {
                st.oacc[nt][m][0] *= alpha;
                st.oacc[nt][m][2] *= alpha;
            }
            st.macc[nt][0] *= alpha;
            st.macc[nt][2] *= alpha;
            st.m_run[nt] = mnew;
        }
    }
}

template <int D, int G, bool VCH0, int NS, int NB, bool MASKED>
__device__ __forceinline__ void pv_accum(const uint32_t (&sb)[NB], int nv, WarpState<D, G> &st, int lane,
                                         const LaneOffsets &o, const float (&s0)[NB][AttendTile<D, G>::NT],
                                         const float (&s1)[NB][AttendTile<D, G>::NT]) {
    using T = AttendTile<D, G>;
    constexpr int NG = T::NG, NT = T::NT;
    constexpr Layout Ly = make_layout(D, 0, NS);
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        // vsa/vsb: scale pairs of tokens (2tig, 2tig+1) and (+8, +9), per scale group
        uint32_t vw[NG], vsa[NS], vsb[NS];
        if constexpr (NG == 4) {
            const uint4 v = ld_s128(sb[b] + o.lane16 + Ly.vc);
            vw[0] = v.x; vw[1] = v.y; vw[2] = v.z; vw[3] = v.w;
        } else {
            const uint2 v = ld_s64(sb[b] + (o.lane16 >> 1) + Ly.vc);
            vw[0] = v.x; vw[1] = v.y;
        }
        if constexpr (NS == 4) {
            const uint32_t a = sb[b] + o.tig16;
            const uint4 x = ld_s128(a + Ly.vs), y = ld_s128(a + Ly.vs + 64);
            vsa[0] = x.x; vsa[1] = x.y; vsa[2] = x.z; vsa[3] = x.w;
            vsb[0] = y.x; vsb[1] = y.y; vsb[2] = y.z; vsb[3] = y.w;
        } else if constexpr (NS == 2) {
            const uint32_t a = sb[b] + (o.tig16 >> 1);
            const uint2 x = ld_s64(a + Ly.vs), y = ld_s64(a + Ly.vs + 32);
            vsa[0] = x.x; vsa[1] = x.y;
            vsb[0] = y.x; vsb[1] = y.y;
        } else {
            const uint32_t a = sb[b] + (o.tig16 >> 2);
            vsa[0] = ld_s32(a + Ly.vs);
            vsb[0] = ld_s32(a + Ly.vs + 16);
        }
        // A rows of the min / denominator / channel-0 product: row g < NS = v-min
        // of scale group g, row NS = ones, row NS+1 = value channel 0 (when protected).
        const uint32_t avm = sb[b] + o.vmin;
        uint32_t vma = (ld_s32(avm + Ly.vm) & o.vmin_mask) | o.ones_lane;
        uint32_t vmb = (ld_s32(avm + Ly.vm + 16 * NS) & o.vmin_mask) | o.ones_lane;
        if constexpr (VCH0) {
            constexpr Layout L1 = make_layout(D, 1, NS);
            const uint32_t a = ld_s32(sb[b] + L1.v0 + tig * 4), c = ld_s32(sb[b] + L1.v0 + 16 + tig * 4);
            if (gid == NS + 1) {
                vma = pack_f16x2(__uint_as_float(a << 16), __uint_as_float(a & 0xffff0000u));
                vmb = pack_f16x2(__uint_as_float(c << 16), __uint_as_float(c & 0xffff0000u));
            }
        }
        if constexpr (MASKED) {
            // rows past the end of the sequence hold stale bytes: zero their factors
            const uint32_t ma = (2 * tig < nv ? 0x0000ffffu : 0u) | (2 * tig + 1 < nv ? 0xffff0000u : 0u);
            const uint32_t mb = (2 * tig + 8 < nv ? 0x0000ffffu : 0u) | (2 * tig + 9 < nv ? 0xffff0000u : 0u);
#pragma unroll
            for (int g = 0; g < NS; ++g) {
                vsa[g] &= ma;
                vsb[g] &= mb;
            }
            vma &= ma;
            vmb &= mb;
        }
        // P~ in the PV B-operand layout (column gid = head gid/2 of the n-tile; odd
        // columns duplicate even ones and are never read back).
        uint32_t pb0[NT], pb1[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float2 e = add2(make_float2(s0[b][nt], s1[b][nt]), make_float2(-st.m_run[nt], -st.m_run[nt]));
            const float p0 = fast_exp2(e.x), p1 = fast_exp2(e.y);
            const uint32_t pp = pack_f16x2(p0, p1);   // lo: token gid, hi: token gid+8
            const uint32_t w0 = __shfl_sync(0xffffffffu, pp, o.srcA);
            const uint32_t w1 = __shfl_sync(0xffffffffu, pp, o.srcA + 4);
            pb0[nt] = prmt(w0, w1, 0x5410u);   // tokens 2tig, 2tig+1
            pb1[nt] = prmt(w0, w1, 0x7632u);   // tokens 2tig+8, 2tig+9
            mma_f16(st.macc[nt], vma, 0u, vmb, 0u, pb0[nt], pb1[nt]);
        }
        if constexpr (NG == 4) {
            // m-tile m is field m of the four words; as fp16 subnormals the
            // fields read code * 4^P * 2^-24 (P = m, or m - 5 after >> 10),
            // undone by vfield_scale when the run is finished
            uint32_t vh[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) vh[k] = vw[k] >> 10;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int gs = NS == 1 ? 0 : g;
                    const uint32_t b0 = hmul2(pb0[nt], vsa[gs]), b1 = hmul2(pb1[nt], vsb[gs]);
#pragma unroll
                    for (int mm = 2 * g; mm < 2 * g + 2; ++mm) {
                        const int P = mm <= 4 ? mm : mm - 5;
                        const uint32_t msk = 0x00030003u << (2 * P);
                        const uint32_t (&src)[4] = mm <= 4 ? vw : vh;
                        mma_f16(st.oacc[nt][mm], src[0] & msk, src[1] & msk, src[2] & msk, src[3] & msk, b0, b1);
                    }
                }
            }
        } else {
#pragma unroll
            for (int w2 = 0; w2 < NG; ++w2) {   // word w2 holds m-tiles 2*w2, 2*w2+1 (= group w2)
                const uint32_t x = vw[w2], xh = x >> 10;
                const uint32_t e0 = code_field<0>(x, xh), e2 = code_field<2>(x, xh);
                const uint32_t e1 = code_field<1>(x, xh), e3 = code_field<3>(x, xh);
                const uint32_t f0 = code_field<4>(x, xh), f2 = code_field<6>(x, xh);
                const uint32_t f1 = code_field<5>(x, xh), f3 = code_field<7>(x, xh);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int gs = NS == 1 ? 0 : w2;
                    const uint32_t b0 = hmul2(pb0[nt], vsa[gs]), b1 = hmul2(pb1[nt], vsb[gs]);
                    mma_f16(st.oacc[nt][2 * w2], e0, e2, e1, e3, b0, b1);
                    mma_f16(st.oacc[nt][2 * w2 + 1], f0, f2, f1, f3, b0, b1);
                }
            }
        }
    }
}

template <int D, int G, bool VCH0, int NS, int NB, bool MASKED>
__device__ __forceinline__ void consume(const uint32_t (&sb)[NB], int nv, WarpState<D, G> &st, int lane,
                                        const LaneOffsets &o) {
    constexpr int NT = AttendTile<D, G>::NT;
    float s0[NB][NT], s1[NB][NT];
    if constexpr (NB > 2) {
        // scores two pages at a time (an odd last page alone): fewer registers
        // live than with all NB at once
#pragma unroll
        for (int h = 0; h + 1 < NB; h += 2) {
            const uint32_t hb[2] = {sb[h], sb[h + 1]};
            float t0[2][NT], t1[2][NT];
            qk_scores<D, G, NS, 2, MASKED>(hb, nv, st, lane, o, t0, t1);
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    s0[h + b][nt] = t0[b][nt];
                    s1[h + b][nt] = t1[b][nt];
                }
        }
        if constexpr (NB % 2 == 1) {
            const uint32_t hb[1] = {sb[NB - 1]};
            float t0[1][NT], t1[1][NT];
            qk_scores<D, G, NS, 1, MASKED>(hb, nv, st, lane, o, t0, t1);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                s0[NB - 1][nt] = t0[0][nt];
                s1[NB - 1][nt] = t1[0][nt];
            }
        }
    } else {
        qk_scores<D, G, NS, NB, MASKED>(sb, nv, st, lane, o, s0, s1);
    }
    max_update<D, G, NB>(st, s0, s1);
    pv_accum<D, G, VCH0, NS, NB, MASKED>(sb, nv, st, lane, o, s0, s1);
}

// Every (run, page slot, kv head) record a consumer warp could own starts
// empty (m = -inf, l = 0): a run shorter than the page slots of a stage
// leaves some warps without a page of it.
__device__ __forceinline__ void init_records(const AttendParams &p, const CtaUnits &cu, int slot_base, int pi,
                                             int jl, int G, int D, int lane) {
    const int R = p.batch * p.nchunks;
    const int u1 = cu.u1;
    int r = cu.r, ur = cu.ur;
    int np = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
    while (r < R && ur < u1) {
        if (np > 0 && lane < G) {
            float *rec = p.part + record_index(slot_base + r, pi, jl, lane, p.pw, p.hc, G) * rec_stride(D);
            rec[0] = -INFINITY;
            rec[1] = 0.0f;
        }
        ur += np;
        ++r;
        np = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
    }
}

// The producer warp of the decode kernels: brings the CTA's units [u0, u1)
// into the ring, pps pages (each hc blocks, one bulk copy) per stage, marks
// which page slots of a stage hold a page, and never leaves with copies in
// flight.  Lane l fills page slots l and l + 32 of a stage (pps <= 64).  The
// page-table entries of the next stage are loaded before the wait for a free
// stage, and checked when their copies are issued.  kEvictFirst: the pages
// are read once per launch, so their copies carry an L2 evict-first policy
// (the packed cache; the BF16 comparison streams without a policy, which
// measured faster for it).  Waits are bounded; a stuck pipeline sets the
// abort flag.
//
// The gate holds back two kinds of copies until the consumers have finished
// the CTA's prologue (its `opened` mbarrier completes once): the first fill
// of the stages from `scratch_first` on, whose memory the prologue works in,
// and, when the same
// launch appends rows to the cache (new_lens non-null), every page at or past
// the first page an append of this call touches.
constexpr int kMaxPagesPerStage = 64;

struct ProducerGate {
    uint64_t *opened;          // completed by the consumers at the end of the CTA's prologue
    int scratch_first;         // first stage used as prologue scratch (>= the stage count: none)
    const int *new_lens;       // rows this launch appends per sequence (null: none)
    const int *seq_before;     // their first position
    int stall;                 // test only: CTA 0 never arms its second stage
    uint64_t wait_ns;          // bound of every wait
};

struct ProducerSlots {
    int phys[2], chunk[2];   // raw page-table entry and kv-head chunk of slot lane + 32k
    bool in[2];              // the slot holds a unit of the CTA that maps to a page-table entry
    bool gated[2];           // the page is written by this launch's append
};

template <bool kEvictFirst>
__device__ __forceinline__ void attend_producer(const AttendParams &p, unsigned char *stage_mem, uint64_t *full,
                                                uint64_t *empty, unsigned char *valid, volatile int *abort_flag,
                                                int S, uint32_t stage_bytes, int kStageBlocks, const CtaUnits &cu,
                                                int iters, int lane, const ProducerGate &gate) {
    const int R = p.batch * p.nchunks;
    const int pps = p.pps;
    const int u0 = cu.u0, u1 = cu.u1;
    if (iters == 0) return;
    if (pps < 1 || pps > kMaxPagesPerStage || pps > kStageBlocks) {   // host plans never do this
        if (lane == 0) {
            *abort_flag = 1;
            dqk_flag_error(kErrBounds);
        }
        return;
    }
    // cursor: run r starts at unit ur and has npr pages; never past the next stage's first unit
    int r = cu.r, ur = cu.ur;
    int npr = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
    const uint32_t copy_bytes = (uint32_t)(p.hc * p.bb);
    const uint64_t stream_policy = kEvictFirst ? l2_policy_evict_first() : 0ull;
    auto fetch = [&](int it) -> ProducerSlots {
        ProducerSlots f;
        const int base = u0 + it * pps;
        int rr = r, st = ur, np = npr;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int slot = 32 * k + lane, u = base + slot;
            f.in[k] = false;
            f.gated[k] = false;
            f.phys[k] = -1;
            f.chunk[k] = 0;
            if (slot < pps && u < u1) {
                while (rr < R && u >= st + np) {
                    st += np;
                    ++rr;
                    np = rr < R ? run_pages(p.seq_lens, p.nchunks, rr) : 0;
                }
                if (rr < R) {
                    const int b = rr / p.nchunks, page = u - st;
                    f.chunk[k] = rr - b * p.nchunks;
                    f.in[k] = true;
                    if (page < p.max_pages) f.phys[k] = p.page_table[(size_t)b * p.max_pages + page];
                    if (gate.new_lens && gate.new_lens[b] > 0) f.gated[k] = page >= gate.seq_before[b] / kPage;
                }
            }
        }
        // the run of the stage's last unit becomes the cursor
        const int last = min(pps, u1 - base) - 1;   // >= 0: stage `it` < iters
        r = __shfl_sync(0xffffffffu, rr, last & 31);
        ur = __shfl_sync(0xffffffffu, st, last & 31);
        npr = __shfl_sync(0xffffffffu, np, last & 31);
        return f;
    };
    ProducerSlots cur = fetch(0);
    int it = 0, stage = 0;
    uint32_t phase = 0;
    bool opened = gate.opened == nullptr;
    for (; it < iters; ++it) {
        ProducerSlots nxt = cur;
        if (it + 1 < iters) nxt = fetch(it + 1);
        int good = 1;
        if (lane == 0) good = mbar_wait_bounded(&empty[stage], phase ^ 1u, gate.wait_ns, 2000u) && !*abort_flag;
        const bool need_open =
            !opened && (stage >= gate.scratch_first || __any_sync(0xffffffffu, cur.gated[0] || cur.gated[1]));
        if (need_open && lane == 0 && good) good = mbar_wait_bounded(gate.opened, 0u, gate.wait_ns, 2000u);
        if (!__shfl_sync(0xffffffffu, good, 0)) {
            if (lane == 0) {
                *abort_flag = 1;
                dqk_flag_error(kErrTimeout);
            }
            break;
        }
        if (need_open) {
            // the prologue's shared-memory scratch and the appended rows (global
            // memory) were written through the generic proxy
            fence_proxy_async_shared();
            fence_proxy_async_global();
            opened = true;
        }
        if (gate.stall && blockIdx.x == 0 && it == 1) {   // test only: this stage is never armed
            cur = nxt;
            if (++stage == S) {
                stage = 0;
                phase ^= 1u;
            }
            continue;
        }
        long long off[2];
        bool have[2];
        unsigned n = 0;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const bool ok = cur.in[k] && cur.phys[k] >= 0 && cur.phys[k] < p.num_pages;
            if (cur.in[k] && !ok) dqk_flag_error(kErrBounds);
            off[k] = ((long long)cur.phys[k] * p.hkv + (long long)cur.chunk[k] * p.hc) * p.bb;
            have[k] = ok;
            n += __popc(__ballot_sync(0xffffffffu, ok));
            const int slot = 32 * k + lane;
            if (slot < pps) valid[stage * kStageBlocks + slot] = ok ? 1 : 0;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(&full[stage], n * copy_bytes);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 2; ++k)
            if (have[k]) {
                void *dst = stage_mem + (size_t)stage * stage_bytes + (size_t)(32 * k + lane) * copy_bytes;
                if constexpr (kEvictFirst) bulk_copy_g2s_hint(dst, p.pool + off[k], copy_bytes, &full[stage], stream_policy);
                else bulk_copy_g2s(dst, p.pool + off[k], copy_bytes, &full[stage]);
            }
        cur = nxt;
        if (++stage == S) {
            stage = 0;
            phase ^= 1u;
        }
    }
    // never leave with copies in flight (exit path: wait, bounded, for the last round of each stage)
    if (lane == 0)
        for (int k = it - 1; k >= 0 && k >= it - S; --k)
            (void)mbar_wait_bounded(&full[k % S], (uint32_t)(k / S) & 1u, gate.wait_ns);
}

// ---------------------------------------------------------------------------
// merge of partial records from n context ranges (one CTA per (sequence,
// query head), one thread per channel): out = sum_r 2^(m_r - M) o_r /
// sum_r 2^(m_r - M) l_r with M = max_r m_r, ranges taken in index order.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(D) k_merge(const float *__restrict__ parts, int n, long long rows,
                                            float *__restrict__ out) {
    const long long row = blockIdx.x;
    const int c = threadIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < n; ++r) M = fmaxf(M, parts[((size_t)r * rows + row) * (D + 2)]);
    float num = 0.0f, den = 0.0f;
    if (M != -INFINITY) {
        for (int r = 0; r < n; ++r) {
            const float *pr = parts + ((size_t)r * rows + row) * (D + 2);
            if (pr[0] == -INFINITY) continue;
            const float w = exp2f(pr[0] - M);
            den = fmaf(w, pr[1], den);
            num = fmaf(w, pr[2 + c], num);
        }
    }
    out[row * D + c] = den > 0.0f ? num / den : 0.0f;
}

}  // namespace dqk
