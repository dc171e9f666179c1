// qprep.cuh -- query transform q' = T_Q q and dynamic channel selection (keep
// channel 0 and the largest-|q'| channels; "Why the cache becomes a
// bottleneck": query-channel pruning; "Throughput on SGLang": 40 % of key
// channels removed from reads), run for the G query heads of one (sequence,
// kv head) by the consumer warps of one CTA in the decode kernel's prologue.
// The kept, scaled q' is laid out as the B operands of the attend loop's
// tensor-core tiles.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace dqk {

// Query fragments of one (sequence, kv head), consumed by the attend loop,
// with qs = q'_c * log2(e)/sqrt(d) on kept channels c >= 1 (0 elsewhere):
//   qf  [B*Hkv][NT][NG][32] uint2      per lane: the two s8x4 registers of the
//       m16n8k32 B operand of group g: rows (channels of the group) 4*tig..+3
//       and 16+4*tig..+3, column n = gid -> query head 4*nt + gid/2; gid even:
//       Q1 = rne(qs/sigma_g), odd: Q2 = clamp(rne((qs/sigma_g - Q1)*256)), so
//       qs ~= sigma_g * (Q1 + Q2/256); sigma_h = (largest |qs| of the head) / 127
//       and sigma_g = sigma_h * 2^-e_g, the smallest such value not below the
//       group's largest |qs| / 127 (the pieces keep 15-16 bits relative to it).
//   qk  [B*Hkv][NT][NG+1][4] float     per head: entry g < NG holds
//       p_g = 2^-e_g / 4^g (the key operand of group g carries code * 4^g), so
//       sigma_g / 4^g = sigma_h * p_g; entry NG holds sigma_h.
//   qm  [B*Hkv][NT][32] uint32         per lane: rows 2*tig, 2*tig+1 of the
//       fp16 min-term B operand, Qsum_{g,h} = sum of qs over the group's kept
//       channels: row k < NG holds the high fp16 part of group k, row NG + k
//       the low part (the key mins repeat in those A columns), so one tile
//       sums both; column 2h holds query head 4*nt + h, odd columns are zero.
//   q0  [B][Hq] float                  qs of channel 0 (always kept).
// Query heads a tile of 4 leaves empty (G < 4) hold zeros everywhere.
struct QueryOut {
    uint2 *qf;
    float *qk;
    uint32_t *qm;
    float *q0;
    int16_t *sel;   // nullable: [B][Hq][n_keep] kept channels, ascending
};

__device__ __forceinline__ uint16_t f16_piece(float x, int piece) {
    const __half hi = __float2half_rn(x);
    if (piece == 0) return __half_as_ushort(hi);
    return __half_as_ushort(__float2half_rn(x - __half2float(hi)));
}

// A [D][D] fp32 transform staged in shared memory by the NTH threads of the
// caller, with coalesced 16-byte loads -- a warp reads 512 contiguous bytes,
// and all of a thread's loads (and the caller's next ones) are in flight
// before its first store -- into rows padded to D*4 + 16 bytes, so that one
// thread per row then reads 16-byte chunks without bank conflicts (eight
// consecutive rows cover the 32 banks).
template <int D>
__host__ __device__ constexpr int pad_row_bytes() { return D * 4 + 16; }

template <int D, int NTH>
struct RowStage {
    static constexpr int Q = D / 4;                     // 16-byte chunks per row
    static constexpr int N = (D * Q + NTH - 1) / NTH;   // chunks per thread
    float4 v[N];
    // asm loads: issued here, in order, ahead of whatever the caller loads next
    __device__ __forceinline__ void load(const float *__restrict__ src, int t) {
        const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const int q = t + i * NTH;
            if (q < D * Q) v[i] = ld_nc_f4(s4 + q);
        }
    }
    __device__ __forceinline__ void store(unsigned char *dst, int t) const {
        const uint32_t base = smem_addr(dst);
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const int q = t + i * NTH;
            if (q < D * Q)
                st_s128(base + (uint32_t)((q / Q) * pad_row_bytes<D>() + (q % Q) * 16),
                        *reinterpret_cast<const uint4 *>(&v[i]));
        }
    }
};

// An input element (fp32 or BF16 storage) as an asm load.
__device__ __forceinline__ float load_elem_vol(const void *p, int dtype, size_t idx) {
    if (dtype == DQK_BF16) return __uint_as_float(ld_u16_vol(reinterpret_cast<const uint16_t *>(p) + idx) << 16);
    return ld_f32_vol(reinterpret_cast<const float *>(p) + idx);
}

// Sum over i ascending of (double)T[row][i] * x[i * xs + n], one fused
// multiply-add after the other for each of the NX vectors (fp32 x fp32
// products are exact in fp64, so the result does not depend on contraction),
// T staged by RowStage.  x is i-major (row stride xs doubles), so the NX
// values of a column come in 16-byte loads.  Eight 16-byte chunks of the row
// per iteration.
template <int D, int NX>
__device__ __forceinline__ void dot_rows_pad(const unsigned char *sT, int row, const double *x, int xs,
                                             double (&acc)[NX]) {
#pragma unroll
    for (int n = 0; n < NX; ++n) acc[n] = 0.0;
    const unsigned char *base = sT + row * pad_row_bytes<D>();
#pragma unroll 1
    for (int k = 0; k < D / 32; ++k) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float4 tv = *reinterpret_cast<const float4 *>(base + (32 * k + 4 * u) * 4);
            const double te[4] = {(double)tv.x, (double)tv.y, (double)tv.z, (double)tv.w};
            const double *xi = x + (32 * k + 4 * u) * xs;
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int n = 0; n < NX; ++n) acc[n] = fma(te[e], xi[e * xs + n], acc[n]);
        }
    }
}

// Shared memory of one query task (16-byte aligned): T_Q[j] in padded rows
// (the q' values [G][D] fp32 reuse it once the sums are done), the query rows
// [D][G] fp64 (i-major), the int8 pieces [G][2][D].
template <int D>
__host__ __device__ constexpr size_t qprep_scratch_bytes(int G) {
    return (size_t)D * pad_row_bytes<D>() + (size_t)G * D * 8 + (size_t)G * 2 * D;
}

// Channels (of this warp's NG per lane, channel 0 excluded) whose magnitude
// bit pattern is >= cand.
template <int NG>
__device__ __forceinline__ int count_ge(const uint32_t (&mag)[NG], bool ch0, uint32_t cand) {
    uint32_t n = 0;
#pragma unroll
    for (int g = 0; g < NG; ++g) n += (mag[g] >= cand && !(g == 0 && ch0)) ? 1u : 0u;
    return (int)__reduce_add_sync(0xffffffffu, n);
}

// The rare paths of the piece arithmetic (subnormal operands), kept out of
// line: the prologue runs once per launch, so its code is fetched cold and
// every inlined instruction costs.
__device__ __noinline__ float ldexp_rare(float x, int e) { return ldexpf(x, e); }
__device__ __noinline__ int exp_offset_rare(float sh, float tg) {
    int e = ilogbf(sh) - ilogbf(tg);
    if (ldexpf(sh, -e) < tg) --e;
    return e;
}

// x * 2^e, exact: an exponent-field addition when x and the result are
// normal, the library function otherwise.
__device__ __forceinline__ float scale_pow2(float x, int e) {
    const uint32_t b = __float_as_uint(x);
    const int ex = (int)((b >> 23) & 0xffu) + e;
    if (((b >> 23) & 0xffu) != 0u && ((b >> 23) & 0xffu) != 0xffu && ex >= 1 && ex <= 254)
        return __uint_as_float((b & 0x807fffffu) | ((uint32_t)ex << 23));
    return ldexp_rare(x, e);
}

// The G query heads of (sequence b, kv head j), by the nthreads threads of
// the calling group (t = 0..nthreads-1; G <= nthreads / 32, D <= nthreads),
// which synchronise on named barrier `bar` (all) and `busy_bar` (the first
// max(D/32, G) warps, which do the work; the others run meanwhile() and
// return):
//   q'_c = fp32(fp64 sequential sum_i T_Q[j][c][i] q_i)   (thread c, all heads);
//   kept = {0} + the n_keep - 1 largest |q'_c| of c >= 1 (fp32 magnitudes,
//   ties to the lower index): warp h selects head h's channels by a bitwise
//   threshold search, then writes head h's fragments and kept channels
//   (ascending).
// meanwhile(): work of the caller's that overlaps the loads of the task.
template <int D, int G, int NTH, typename Meanwhile>
__device__ void qprep_kv(const float *__restrict__ t_q, const void *__restrict__ q, int dtype, int hq, int hkv, int pct,
                         float qscale, int b, int j, int t, int bar, int busy_bar, unsigned char *scratch,
                         const QueryOut &qo, Meanwhile meanwhile) {
    constexpr int NG = D / 32;
    constexpr int NT = G > 4 ? 2 : 1;
    constexpr int nthreads = NTH;
    const int warp = t >> 5, lane = t & 31;
    const int nk = keep_count(D, pct);
    double *qin = reinterpret_cast<double *>(scratch + (size_t)D * pad_row_bytes<D>());
    signed char *q8 = reinterpret_cast<signed char *>(qin + (size_t)G * D);
    float *qpv = reinterpret_cast<float *>(scratch);   // [G][D] after the sums

    // stage T_Q[j] and the G query rows (query h, channel c -> qin[c][h]):
    // every load in flight before the first store
    named_bar_sync(bar, nthreads);   // the previous task is done with the scratch
    RowStage<D, NTH> rows;
    rows.load(t_q + (size_t)j * D * D, t);
    constexpr int QN = (G * D + NTH - 1) / NTH;
    const size_t qbase = ((size_t)b * hq + (size_t)j * G) * D;
    float qv[QN];
#pragma unroll
    for (int k = 0; k < QN; ++k)
        if (t + k * NTH < G * D) qv[k] = load_elem_vol(q, dtype, qbase + t + k * NTH);
    rows.store(scratch, t);
#pragma unroll
    for (int k = 0; k < QN; ++k) {
        const int i = t + k * NTH;
        if (i < G * D) qin[(i % D) * G + i / D] = (double)qv[k];
    }
    named_bar_sync(bar, nthreads);   // T_Q[j] and the query rows are in
    // the warps the task leaves idle run the caller's `meanwhile` work
    constexpr int kBusy = (D / 32 > G ? D / 32 : G);
    if (warp >= kBusy) {
        meanwhile();
        return;
    }

    // q'_c of every head: G interleaved sums per thread (thread c = row c),
    // ascending i, exact fp32 x fp32 products accumulated in fp64, one
    // rounding each
    double acc[G];
    if (t < D) dot_rows_pad<D, G>(scratch, t, qin, G, acc);
    named_bar_sync(busy_bar, 32 * kBusy);   // T_Q is dead
    if (t < D) {
#pragma unroll
        for (int n = 0; n < G; ++n) qpv[n * D + t] = __double2float_rn(acc[n]);
    }
    named_bar_sync(busy_bar, 32 * kBusy);

    if (warp < G) {
        const int h = warp, hl = h, nt = hl >> 2, hh = hl & 3;
        const int hg = j * G + h;   // query head index
        // selection of the nk - 1 channels c >= 1 with the largest |q'_c|
        // (fp32 magnitudes as bit patterns), ties to the lower index; lane owns
        // channels lane + 32 g.  T = the (nk-1)-th largest magnitude, found bit
        // by bit from the top (the largest T with at least nk - 1 magnitudes >=
        // T); then every channel above T is kept, and of those equal to T the
        // lowest-indexed ones that complete the count.
        const int m = nk - 1;
        uint32_t mag[NG];
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const int c = lane + 32 * g;
            mag[g] = c == 0 ? 0u : (__float_as_uint(qpv[h * D + c]) & 0x7fffffffu);
        }
        const bool ch0 = lane == 0;   // channel 0 (g = 0) takes no part
        uint32_t T = 0;
        int cnt = D - 1;   // channels >= T
        // bit 30 alone, then two bits per step (three candidates counted at
        // once); done as soon as exactly m channels are >= T (the prefix then
        // separates the kept channels from the others)
        {
            const int n = count_ge<NG>(mag, ch0, 1u << 30);
            if (n >= m) {
                T = 1u << 30;
                cnt = n;
            }
        }
#pragma unroll 1
        for (int bit = 28; bit >= 0 && cnt != m; bit -= 2) {
            const int n3 = count_ge<NG>(mag, ch0, T | (3u << bit)), n2 = count_ge<NG>(mag, ch0, T | (2u << bit)),
                      n1 = count_ge<NG>(mag, ch0, T | (1u << bit));
            const uint32_t d = n3 >= m ? 3u : n2 >= m ? 2u : n1 >= m ? 1u : 0u;
            T |= d << bit;
            cnt = d == 3u ? n3 : d == 2u ? n2 : d == 1u ? n1 : cnt;
        }
        // with cnt > m, T is the m-th largest magnitude itself and ties at T
        // go to the lower channel indices
        const bool exact = cnt == m;
        int need = exact ? 0 : m - (T == 0x7fffffffu ? 0 : count_ge<NG>(mag, ch0, T + 1u));
        uint32_t kmask[NG];
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const bool eq = !exact && mag[g] == T && !(g == 0 && ch0) && m > 0;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const int rank = __popc(eqm & ((1u << lane) - 1u));   // equal channels of lower index in this group
            const bool above = exact ? mag[g] >= T : mag[g] > T;
            const bool keep = (above && !(g == 0 && ch0) && m > 0) || (eq && rank < need);
            kmask[g] = __ballot_sync(0xffffffffu, keep);
            need -= __popc(eqm);
        }
        kmask[0] |= 1u;   // channel 0 is always kept

        // lane owns channels lane + 32 g: scaled q' on kept channels >= 1, group
        // sums and maxima, sigma_h, and the two int8 pieces relative to sigma_g =
        // sigma_h * 2^-e, the smallest such value not below the group's largest
        // |qs| / 127, so that sigma_g / sigma_h is a power of two
        float qs[NG], v[NG], gs[NG], gm[NG];
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const int c = lane + 32 * g;
            qs[g] = qpv[h * D + c] * qscale;
            v[g] = (((kmask[g] >> lane) & 1u) && c != 0) ? qs[g] : 0.0f;
            gs[g] = v[g];
            gm[g] = fabsf(v[g]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                gs[g] += __shfl_xor_sync(0xffffffffu, gs[g], o);
                gm[g] = fmaxf(gm[g], __shfl_xor_sync(0xffffffffu, gm[g], o));
            }
        }
        float hm = 0.0f;
#pragma unroll
        for (int g = 0; g < NG; ++g) hm = fmaxf(hm, gm[g]);
        constexpr float kInv127 = 1.0f / 127.0f;
        const float sh = hm * kInv127;
        const float rsh = sh > 0.0f ? 1.0f / sh : 0.0f;   // 1 / sigma_g = 2^e / sh
        float sig[NG];
        int before = 0;   // kept channels in earlier groups
        const uint32_t shb = __float_as_uint(sh);
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            // sigma_g = sh * 2^-e with e >= 0 the largest such that sigma_g >= tg:
            // sh = 2^Es ms, tg = 2^Et mt (normal, ms, mt in [1, 2)) give
            // e = Es - Et - [ms < mt]; exponent-field arithmetic, the library
            // functions for the rare subnormal operand
            const float tg = gm[g] * kInv127;
            const uint32_t tgb = __float_as_uint(tg);
            int e = 0;
            if (tg > 0.0f) {
                if ((shb >> 23) != 0u && (tgb >> 23) != 0u) {
                    e = (int)(shb >> 23) - (int)(tgb >> 23) - ((shb & 0x7fffffu) < (tgb & 0x7fffffu) ? 1 : 0);
                } else {
                    e = exp_offset_rare(sh, tg);
                }
            }
            int q1 = 0, q2 = 0;
            if (sh > 0.0f) {
                const float x = v[g] * scale_pow2(rsh, e);   // v / sigma_g
                q1 = max(-127, min(127, __float2int_rn(x)));
                q2 = max(-128, min(127, __float2int_rn((x - (float)q1) * 256.0f)));
            }
            // p_g = 2^(-e - 2g), a normal number unless the query is degenerate
            const int pe = 127 - e - 2 * g;
            sig[g] = pe >= 1 ? __uint_as_float((uint32_t)pe << 23) : ldexp_rare(1.0f, -e - 2 * g);
            const int c = lane + 32 * g;
            q8[(h * 2 + 0) * D + c] = (signed char)q1;
            q8[(h * 2 + 1) * D + c] = (signed char)q2;
            // kept channels ascending: earlier groups, then lanes below
            if (qo.sel && ((kmask[g] >> lane) & 1u))
                qo.sel[((size_t)b * hq + hg) * nk + before + __popc(kmask[g] & ((1u << lane) - 1u))] = (int16_t)c;
            before += __popc(kmask[g]);
        }
        if (lane == 0) qo.q0[(size_t)b * hq + hg] = qs[0];
        __syncwarp();

        // this head's lanes of the fragments: 8 lanes (gid = 2 hh + piece) per group
        const size_t bj = (size_t)b * hkv + j;
        for (int idx = lane; idx < 8 * NG; idx += 32) {
            const int L = 8 * hh + (idx & 7), gg = idx >> 3;
            const int gid = L >> 2, tig = L & 3, piece = gid & 1;
            const unsigned char *r = reinterpret_cast<const unsigned char *>(&q8[(h * 2 + piece) * D + 32 * gg]);
            uint32_t w0 = 0, w1 = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                w0 |= (uint32_t)r[4 * tig + i] << (8 * i);
                w1 |= (uint32_t)r[16 + 4 * tig + i] << (8 * i);
            }
            qo.qf[((bj * NT + nt) * NG + gg) * 32 + L] = make_uint2(w0, w1);
        }
#pragma unroll
        for (int g = 0; g <= NG; ++g)
            if (lane == g) qo.qk[((bj * NT + nt) * (NG + 1) + g) * 4 + hh] = g < NG ? sig[g] : sh;
        if (lane < 8) {
            const int L = 8 * hh + lane, gid = L >> 2, tig = L & 3;
            uint32_t w = 0;
            if ((gid & 1) == 0) {
                // rows k = 2*tig, 2*tig + 1: piece k / NG (0 high, 1 low) of group k % NG
                const int k0 = 2 * tig, k1 = 2 * tig + 1;
                float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    if (k0 % NG == g) s0 = gs[g];
                    if (k1 % NG == g) s1 = gs[g];
                }
                const uint32_t r0 = k0 < 2 * NG ? f16_piece(s0, k0 / NG) : 0u;
                const uint32_t r1 = k1 < 2 * NG ? f16_piece(s1, k1 / NG) : 0u;
                w = r0 | (r1 << 16);
            }
            qo.qm[(bj * NT + nt) * 32 + L] = w;
        }
        // the head slots of a 4-head tile that no query head fills (G < 4)
        if (G < 4 && h == 0) {
            for (int idx = lane; idx < (4 - G) * 8 * (NG + 2); idx += 32) {
                const int hs = G + idx / (8 * (NG + 2)), rem = idx % (8 * (NG + 2));
                const int L = 8 * hs + (rem & 7), part = rem >> 3;   // part < NG: qf of group part
                if (part < NG) qo.qf[((bj * NT) * NG + part) * 32 + L] = make_uint2(0u, 0u);
                else if (part == NG) qo.qm[(bj * NT) * 32 + L] = 0u;
                else if ((rem & 7) <= NG) qo.qk[((bj * NT) * (NG + 1) + (rem & 7)) * 4 + hs] = 0.0f;
            }
        }
    }
}

}  // namespace dqk
