// attend.cuh -- k_attend: split-K pruned-channel attention over the INT2 paged
// cache ("Throughput on SGLang": pruning removes 40 % of key channels from
// reads, quantization cuts storage to 2 bits per value), and k_combine, the
// cross-split log-sum-exp merge.
//
// Work split: the cache is a sequence of units (pages of one run; a run is a
// (sequence, chunk of <= 8 kv heads)).  CTA c of C owns units
// [floor(c*U/C), floor((c+1)*U/C)): every CTA streams the same number of pages
// whatever the length mix.  A producer warp brings whole units in with 1-D bulk
// async copies (one copy = 16 tokens x up to 8 kv heads, contiguous) into a
// ring of `stages` shared-memory buffers guarded by mbarriers; 8 consumer
// warps, one per (kv head, page slot), run the tensor-core math.
//
// Per consumer warp and page (16 tokens x G query heads), with
// qs = q' * log2(e)/sqrt(d) on the kept channels:
//   QK   D_g[t, n] = sum_{c in g} code[t, c] * qs_hilo[c, n]     (m16n8k16, per group)
//        n = (head, fp16 high/low part of qs): the hi/lo split uses the columns
//        a GQA group of 4 leaves free, so q is carried at ~22 bits;
//        s[t, h] = sum_g scale[t, g] * (D_g[t,(h,hi)] + D_g[t,(h,lo)])
//                + sum_g min[t, g] * Qsum[g, h]   (one extra m16n8k16)
//                + qs_0[h] * k0[t]                (BF16 channel 0, fp32)
//   online softmax in base 2 (running max per head, exact rescale on growth)
//   PV   O^T[c, h] += sum_t code_v[t, c] * (p~[t, h] * vscale[t, g(c)])
//        with p~ = fp16(p); one extra m16n8k16 gives sum_t p~ * vmin[t, g] and
//        l = sum_t p~ (a row of ones), so numerator and denominator see the
//        same rounded weights.
// Codes become exact fp16 operands with one LOP3 and one HSUB2 per pair.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace dqk {

constexpr int kConsumerWarps = 8;
constexpr int kAttendThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxStages = 16;
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s: a stuck pipeline reports DQK_ERR_TIMEOUT

struct AttendParams {
    const uint8_t *pool;
    long long num_pages;
    const int *seq_lens;
    const int *page_table;
    const uint2 *qf;
    const uint32_t *qm;
    const float *q0;
    float *part;
    int batch, hq, hkv, hc, pps, nchunks, max_pages, bb, v_ch0, stages, num_ctas;
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

__device__ __forceinline__ size_t record_index(int slot, int ps, int jl, int hh, int pps, int hc, int G) {
    return (((size_t)slot * pps + ps) * hc + jl) * G + hh;
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

template <int D, int G>
__global__ void __launch_bounds__(kAttendThreads, 1) k_attend(const AttendParams p) {
    using T = AttendTile<D, G>;
    constexpr int NG = T::NG, NT = T::NT, NM = T::NM;
    extern __shared__ __align__(128) unsigned char attend_smem[];
    unsigned char *smem_raw = attend_smem;
    const int S = p.stages;
    const uint32_t stage_bytes = (uint32_t)(kConsumerWarps * p.bb);
    unsigned char *stage_mem = smem_raw;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem_raw + (size_t)S * stage_bytes);
    uint64_t *empty = full + S;
    unsigned char *valid = reinterpret_cast<unsigned char *>(empty + S);   // [S][8]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(valid + S * 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = p.batch * p.nchunks;
    const long long C = p.num_ctas;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const long long U = warp_total_units(p.seq_lens, p.nchunks, R, lane);
    const long long u0 = (long long)blockIdx.x * U / C, u1 = ((long long)blockIdx.x + 1) * U / C;
    const long long nunits = u1 - u0;
    const int iters = (int)((nunits + p.pps - 1) / p.pps);

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        // Let the next kernel in the stream start its prologue early.
        grid_dependents_launch();
        if (iters == 0) return;
        int r;
        long long ur;
        warp_locate(p.seq_lens, p.nchunks, R, u0, lane, r, ur);
        int npr = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
        const uint32_t copy_bytes = (uint32_t)(p.hc * p.bb);
        // byte offset in the pool of unit ubase + lane, or -1
        auto fetch = [&](long long ubase, int &r_c, long long &ur_c, int &np_c) -> long long {
            const long long u = ubase + lane;
            int rr = r_c;
            long long st = ur_c;
            int np = np_c;
            while (rr < R && u >= st + np) {
                st += np;
                ++rr;
                np = rr < R ? run_pages(p.seq_lens, p.nchunks, rr) : 0;
            }
            long long off = -1;
            if (u < u1 && rr < R) {
                const int b = rr / p.nchunks, chunk = rr % p.nchunks;
                const long long page = u - st;
                if (page < p.max_pages) {
                    const int phys = p.page_table[(size_t)b * p.max_pages + page];
                    if (phys >= 0 && phys < p.num_pages)
                        off = ((long long)phys * p.hkv + (long long)chunk * p.hc) * p.bb;
                }
                if (off < 0) dqk_flag_error(kErrBounds);
            }
            // advance the warp cursor to the run of unit ubase + 32
            rr = __shfl_sync(0xffffffffu, rr, 31);
            st = __shfl_sync(0xffffffffu, st, 31);
            np = __shfl_sync(0xffffffffu, np, 31);
            r_c = rr;
            ur_c = st;
            np_c = np;
            return off;
        };
        long long off_next = fetch(u0, r, ur, npr);
        bool ok = true;
        int it = 0;
        for (long long ubase = u0; ubase < u1 && ok; ubase += 32) {
            const long long off_cur = off_next;
            if (ubase + 32 < u1) off_next = fetch(ubase + 32, r, ur, npr);
            // stage iterations whose units lie in this batch of 32
            for (; ok && (long long)it * p.pps < nunits && u0 + (long long)it * p.pps < ubase + 32; ++it) {
                const int s = it % S;
                const uint32_t round = (uint32_t)(it / S);
                int good = 1;
                if (lane == 0) good = mbar_wait_bounded(&empty[s], (round & 1u) ^ 1u, kWaitLimitNs) && !*abort_flag;
                good = __shfl_sync(0xffffffffu, good, 0);
                if (!good) {
                    if (lane == 0) {
                        *abort_flag = 1;
                        dqk_flag_error(kErrTimeout);
                    }
                    ok = false;
                    break;
                }
                uint32_t bytes = 0;
                long long offs[8];
#pragma unroll
                for (int ps = 0; ps < 8; ++ps) {
                    const long long u = u0 + (long long)it * p.pps + ps;
                    const int src = (int)(u - ubase);
                    long long o = __shfl_sync(0xffffffffu, off_cur, src & 31);
                    if (ps >= p.pps || u >= u1) o = -1;
                    offs[ps] = o;
                    if (o >= 0) bytes += copy_bytes;
                }
                if (lane == 0) {
#pragma unroll
                    for (int ps = 0; ps < 8; ++ps)
                        if (ps < p.pps) valid[s * 8 + ps] = offs[ps] >= 0 ? 1 : 0;
                    mbar_arrive_expect_tx(&full[s], bytes);
#pragma unroll
                    for (int ps = 0; ps < 8; ++ps)
                        if (ps < p.pps && offs[ps] >= 0)
                            bulk_copy_g2s(stage_mem + (size_t)s * stage_bytes + (size_t)ps * copy_bytes,
                                          p.pool + offs[ps], copy_bytes, &full[s]);
                }
            }
        }
        // never leave with copies in flight: wait (bounded) for the last round of each stage
        if (lane == 0) {
            const int issued = it;
            for (int k = issued - 1; k >= 0 && k >= issued - S; --k)
                (void)mbar_wait_bounded(&full[k % S], (uint32_t)(k / S) & 1u, kWaitLimitNs);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int jl = warp % p.hc, ps = warp / p.hc;
    const int gid = lane >> 2, tig = lane & 3;
    const int slot_base = (int)blockIdx.x;

    // Every (run, page slot, kv head) record this warp could own starts empty:
    // a run shorter than the page slots leaves some warps without a page.
    if (nunits > 0 && ps < p.pps) {
        int r;
        long long ur;
        warp_locate(p.seq_lens, p.nchunks, R, u0, lane, r, ur);
        int np = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
        while (r < R && ur < u1) {
            if (np > 0 && lane < G) {
                float *rec = p.part + record_index(slot_base + r, ps, jl, lane, p.pps, p.hc, G) * (2 + D);
                rec[0] = -INFINITY;
                rec[1] = 0.0f;
            }
            ur += np;
            ++r;
            np = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
        }
    }
    if (iters == 0) return;
    grid_dependency_wait();     // query fragments come from k_qprep

    int r;
    long long ur;
    warp_locate(p.seq_lens, p.nchunks, R, u0, lane, r, ur);
    int npr = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
    int cur_run = -1, Lb = 0;

    uint2 qb[NT][NG][2];
    uint32_t qmin[NT];
    float q0v[NT], m_run[NT];
    float oacc[NT][NM][4];
    float macc[NT][4];

    auto start_run = [&](int rr) {
        const int b = rr / p.nchunks, chunk = rr % p.nchunks;
        const int j = chunk * p.hc + jl;
        const size_t bj = (size_t)b * p.hkv + j;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int g = 0; g < NG; ++g)
#pragma unroll
                for (int s = 0; s < 2; ++s) qb[nt][g][s] = p.qf[(((bj * NT + nt) * NG + g) * 2 + s) * 32 + lane];
            qmin[nt] = p.qm[(bj * NT + nt) * 32 + lane];
            const int hh = 4 * nt + tig;
            q0v[nt] = hh < G ? p.q0[(size_t)b * p.hq + j * G + hh] : 0.0f;
            m_run[nt] = -INFINITY;
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int e = 0; e < 4; ++e) oacc[nt][m][e] = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; ++e) macc[nt][e] = 0.0f;
        }
        Lb = p.seq_lens[b];
        cur_run = rr;
    };

    auto finish_run = [&](int rr) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float minterm[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g) minterm[g] = __shfl_sync(0xffffffffu, macc[nt][0], g * 4 + tig);
            const float l = __shfl_sync(0xffffffffu, macc[nt][0], NG * 4 + tig);
            const float v0t = __shfl_sync(0xffffffffu, macc[nt][0], (NG + 1) * 4 + tig);
            const int hh = 4 * nt + tig;
            if (hh < G) {
                float *rec = p.part + record_index(slot_base + rr, ps, jl, hh, p.pps, p.hc, G) * (2 + D);
                if (gid == 0) {
                    rec[0] = m_run[nt];
                    rec[1] = l;
                }
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    const int c0 = 16 * m + gid, c1 = c0 + 8;
                    const float mt = minterm[m >> 1];
                    rec[2 + c0] = (p.v_ch0 && c0 == 0) ? v0t : oacc[nt][m][0] + mt;
                    rec[2 + c1] = oacc[nt][m][2] + mt;
                }
            }
        }
    };

    const uint32_t kOnes = 0x3C003C00u;
    bool ok = true;
    for (int it = 0; it < iters; ++it) {
        const int s = it % S;
        const uint32_t round = (uint32_t)(it / S);
        if (!mbar_wait_bounded(&full[s], round & 1u, kWaitLimitNs) || *abort_flag) {
            if (lane == 0) {
                *abort_flag = 1;
                dqk_flag_error(kErrTimeout);
            }
            ok = false;
            break;
        }
        const long long u = u0 + (long long)it * p.pps + ps;
        if (ps < p.pps && u < u1) {
            while (r < R && u >= ur + npr) {
                ur += npr;
                ++r;
                npr = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
            }
            if (r != cur_run) {
                if (cur_run >= 0) finish_run(cur_run);
                start_run(r);
            }
            if (valid[s * 8 + ps]) {
                const long long page = u - ur;
                const int nv = (int)min((long long)kPage, (long long)Lb - page * kPage);
                const unsigned char *blk = stage_mem + (size_t)s * stage_bytes + (size_t)(ps * p.hc + jl) * p.bb;
                const Layout Ly = make_layout(D, p.v_ch0);

                // ------------------------------------------------ key side
                uint32_t kw[NG];
                if constexpr (NG == 4) {
                    const uint4 v = lds128(blk + Ly.kc + lane * 16);
                    kw[0] = v.x; kw[1] = v.y; kw[2] = v.z; kw[3] = v.w;
                } else {
                    const uint2 v = lds64(blk + Ly.kc + lane * 8);
                    kw[0] = v.x; kw[1] = v.y;
                }
                uint32_t ks0[(NG + 1) / 2], ks1[(NG + 1) / 2];   // fp16 scale pairs of tokens gid, gid+8
                if constexpr (NG == 4) {
                    const uint2 a = lds64(blk + Ly.ks + gid * 8), c = lds64(blk + Ly.ks + (gid + 8) * 8);
                    ks0[0] = a.x; ks0[1] = a.y; ks1[0] = c.x; ks1[1] = c.y;
                } else {
                    ks0[0] = lds32(blk + Ly.ks + gid * 4);
                    ks1[0] = lds32(blk + Ly.ks + (gid + 8) * 4);
                }
                const bool has_min = tig < NG / 2;
                const uint32_t km0 = has_min ? lds32(blk + Ly.km + gid * 2 * NG + tig * 4) : 0u;
                const uint32_t km1 = has_min ? lds32(blk + Ly.km + (gid + 8) * 2 * NG + tig * 4) : 0u;
                const uint32_t k0w = lds32(blk + Ly.k0 + gid * 4);
                const float k0a = __uint_as_float(k0w << 16), k0b = __uint_as_float(k0w & 0xffff0000u);

                uint32_t ka[NG][2][4];
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    const uint32_t x = kw[g], xh = x >> 10;
                    ka[g][0][0] = code_field<0>(x, xh);
                    ka[g][0][1] = code_field<1>(x, xh);
                    ka[g][0][2] = code_field<2>(x, xh);
                    ka[g][0][3] = code_field<3>(x, xh);
                    ka[g][1][0] = code_field<4>(x, xh);
                    ka[g][1][1] = code_field<5>(x, xh);
                    ka[g][1][2] = code_field<6>(x, xh);
                    ka[g][1][3] = code_field<7>(x, xh);
                }

                float p0[NT], p1[NT], alpha[NT];
                bool grow = false;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float cm[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_f16(cm, km0, km1, 0u, 0u, qmin[nt], 0u);
                    float s0 = cm[0] + cm[1], s1 = cm[2] + cm[3];
#pragma unroll
                    for (int g = 0; g < NG; ++g) {
                        float dg[4] = {0.f, 0.f, 0.f, 0.f};
                        mma_f16(dg, ka[g][0][0], ka[g][0][1], ka[g][0][2], ka[g][0][3], qb[nt][g][0].x,
                                qb[nt][g][0].y);
                        mma_f16(dg, ka[g][1][0], ka[g][1][1], ka[g][1][2], ka[g][1][3], qb[nt][g][1].x,
                                qb[nt][g][1].y);
                        const float2 sa = f16x2_to_f32x2(ks0[g >> 1]), sb = f16x2_to_f32x2(ks1[g >> 1]);
                        s0 = fmaf((g & 1) ? sa.y : sa.x, dg[0] + dg[1], s0);
                        s1 = fmaf((g & 1) ? sb.y : sb.x, dg[2] + dg[3], s1);
                    }
                    s0 = fmaf(q0v[nt], k0a, s0);
                    s1 = fmaf(q0v[nt], k0b, s1);
                    if (gid >= nv) s0 = -INFINITY;
                    if (gid + 8 >= nv) s1 = -INFINITY;
                    float mx = fmaxf(s0, s1);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    const float mnew = fmaxf(m_run[nt], mx);
                    grow |= mnew > m_run[nt];
                    const float mref = mnew == -INFINITY ? 0.0f : mnew;
                    alpha[nt] = exp2f(m_run[nt] - mref);
                    p0[nt] = exp2f(s0 - mref);
                    p1[nt] = exp2f(s1 - mref);
                    m_run[nt] = mnew;
                }
                if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                        for (int m = 0; m < NM; ++m) {
                            oacc[nt][m][0] *= alpha[nt];
                            oacc[nt][m][2] *= alpha[nt];
                        }
                        macc[nt][0] *= alpha[nt];
                        macc[nt][2] *= alpha[nt];
                    }
                }

                // ------------------------------------------------ value side
                uint32_t vw[NG];
                if constexpr (NG == 4) {
                    const uint4 v = lds128(blk + Ly.vc + lane * 16);
                    vw[0] = v.x; vw[1] = v.y; vw[2] = v.z; vw[3] = v.w;
                } else {
                    const uint2 v = lds64(blk + Ly.vc + lane * 8);
                    vw[0] = v.x; vw[1] = v.y;
                }
                uint32_t vsa[NG], vsb[NG];   // scale pairs of tokens (2tig, 2tig+1) and (2tig+8, 2tig+9)
                if constexpr (NG == 4) {
                    const uint4 a = lds128(blk + Ly.vs + tig * 16), c = lds128(blk + Ly.vs + (tig + 4) * 16);
                    vsa[0] = a.x; vsa[1] = a.y; vsa[2] = a.z; vsa[3] = a.w;
                    vsb[0] = c.x; vsb[1] = c.y; vsb[2] = c.z; vsb[3] = c.w;
                } else {
                    const uint2 a = lds64(blk + Ly.vs + tig * 8), c = lds64(blk + Ly.vs + (tig + 4) * 8);
                    vsa[0] = a.x; vsa[1] = a.y;
                    vsb[0] = c.x; vsb[1] = c.y;
                }
                uint32_t vma = 0u, vmb = 0u;    // rows of the min / ones / channel-0 product
                if (gid < NG) {
                    vma = lds32(blk + Ly.vm + (tig * NG + gid) * 4);
                    vmb = lds32(blk + Ly.vm + ((tig + 4) * NG + gid) * 4);
                } else if (gid == NG) {
                    vma = kOnes;
                    vmb = kOnes;
                } else if (gid == NG + 1 && p.v_ch0) {
                    const uint32_t a = lds32(blk + Ly.v0 + tig * 4), c = lds32(blk + Ly.v0 + (tig + 4) * 4);
                    vma = pack_f16x2(__uint_as_float(a << 16), __uint_as_float(a & 0xffff0000u));
                    vmb = pack_f16x2(__uint_as_float(c << 16), __uint_as_float(c & 0xffff0000u));
                }
                if (nv < kPage) {
                    // rows past the end of the sequence hold stale bytes: zero their weights' factors
                    const uint32_t ma = (2 * tig < nv ? 0x0000ffffu : 0u) | (2 * tig + 1 < nv ? 0xffff0000u : 0u);
                    const uint32_t mb = (2 * tig + 8 < nv ? 0x0000ffffu : 0u) | (2 * tig + 9 < nv ? 0xffff0000u : 0u);
#pragma unroll
                    for (int g = 0; g < NG; ++g) {
                        vsa[g] &= ma;
                        vsb[g] &= mb;
                    }
                    vma &= ma;
                    vmb &= mb;
                }

                // P~ in the PV B-operand layout: column gid (even) = head gid/2 of the n-tile
                uint32_t pb0[NT], pb1[NT];
                const int srcA = (2 * tig) * 4 + (gid >> 1), srcB = srcA + 4;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint32_t pp = pack_f16x2(p0[nt], p1[nt]);   // lo: token gid, hi: token gid+8
                    const uint32_t w0 = __shfl_sync(0xffffffffu, pp, srcA);
                    const uint32_t w1 = __shfl_sync(0xffffffffu, pp, srcB);
                    pb0[nt] = (gid & 1) ? 0u : prmt(w0, w1, 0x5410u);   // tokens 2tig, 2tig+1
                    pb1[nt] = (gid & 1) ? 0u : prmt(w0, w1, 0x7632u);   // tokens 2tig+8, 2tig+9
                    mma_f16(macc[nt], vma, 0u, vmb, 0u, pb0[nt], pb1[nt]);
                }
#pragma unroll
                for (int w2 = 0; w2 < NG; ++w2) {       // word w2 holds m-tiles 2*w2 and 2*w2+1 (= group w2)
                    const uint32_t x = vw[w2], xh = x >> 10;
                    const uint32_t e0 = code_field<0>(x, xh), e2 = code_field<2>(x, xh);
                    const uint32_t e1 = code_field<1>(x, xh), e3 = code_field<3>(x, xh);
                    const uint32_t f0 = code_field<4>(x, xh), f2 = code_field<6>(x, xh);
                    const uint32_t f1 = code_field<5>(x, xh), f3 = code_field<7>(x, xh);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint32_t b0 = hmul2(pb0[nt], vsa[w2]), b1 = hmul2(pb1[nt], vsb[w2]);
                        mma_f16(oacc[nt][2 * w2], e0, e2, e1, e3, b0, b1);
                        mma_f16(oacc[nt][2 * w2 + 1], f0, f2, f1, f3, b0, b1);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (ok && cur_run >= 0) finish_run(cur_run);
}

// ---------------------------------------------------------------------------
// log-sum-exp combine: out[b][h] = sum_i o_i 2^(m_i - m*) / sum_i l_i 2^(m_i - m*)
// over the records of every CTA (and page slot) that held pages of (b, h).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) k_combine(const int *__restrict__ seq_lens, int batch, int hq, int hkv,
                                                 int hc, int pps, int nchunks, int num_ctas,
                                                 const float *__restrict__ part, float *__restrict__ out) {
    __shared__ long long sh_U, sh_ur;
    __shared__ int sh_np;
    const int h = blockIdx.x, b = blockIdx.y;
    const int G = hq / hkv, j = h / G, chunk = j / hc, jl = j % hc, hh = h % G;
    const int r = b * nchunks + chunk, R = batch * nchunks;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const long long U = warp_total_units(seq_lens, nchunks, R, lane);
        long long base = 0;   // start unit of run r
        for (int r0 = 0; r0 < r; r0 += 32) {
            const int rr = r0 + lane;
            long long np = rr < r ? run_pages(seq_lens, nchunks, rr) : 0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) np += __shfl_xor_sync(0xffffffffu, np, o);
            base += np;
        }
        if (lane == 0) {
            sh_U = U;
            sh_ur = base;
            sh_np = run_pages(seq_lens, nchunks, r);
        }
    }
    __syncthreads();
    grid_dependency_wait();     // partial records come from k_attend
    const long long U = sh_U, ur = sh_ur;
    const int np = sh_np;
    float *o = out + ((size_t)b * hq + h) * D;
    if (np == 0) {
        for (int c = threadIdx.x; c < D; c += blockDim.x) o[c] = 0.0f;
        return;
    }
    const int cf = (int)cta_of_unit(ur, U, num_ctas), cl = (int)cta_of_unit(ur + np - 1, U, num_ctas);
    // CTAs with an empty unit range (more CTAs than units) wrote no records
    auto has_units = [&](int c) { return (long long)c * U / num_ctas < ((long long)c + 1) * U / num_ctas; };
    float mstar = -INFINITY;
    for (int c = cf; c <= cl; ++c)
        if (has_units(c))
            for (int s = 0; s < pps; ++s)
                mstar = fmaxf(mstar, part[record_index(c + r, s, jl, hh, pps, hc, G) * (2 + D)]);
    float den = 0.0f;
    for (int c = cf; c <= cl; ++c)
        if (has_units(c))
            for (int s = 0; s < pps; ++s) {
            const float *rec = part + record_index(c + r, s, jl, hh, pps, hc, G) * (2 + D);
            if (rec[0] != -INFINITY) den += rec[1] * exp2f(rec[0] - mstar);
        }
    for (int ch = threadIdx.x; ch < D; ch += blockDim.x) {
        float num = 0.0f;
        for (int c = cf; c <= cl; ++c)
            if (has_units(c))
                for (int s = 0; s < pps; ++s) {
                const float *rec = part + record_index(c + r, s, jl, hh, pps, hc, G) * (2 + D);
                if (rec[0] != -INFINITY) num += rec[2 + ch] * exp2f(rec[0] - mstar);
            }
        o[ch] = den > 0.0f ? num / den : 0.0f;
    }
}

}  // namespace dqk
