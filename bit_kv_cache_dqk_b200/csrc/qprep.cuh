// qprep.cuh -- k_qprep: query transform q' = T_Q q and dynamic channel
// selection (keep channel 0 and the largest-|q'| channels; "Why the cache
// becomes a bottleneck": query-channel pruning; "Throughput on SGLang": 40 %
// of key channels removed from reads).  One CTA per (sequence, kv head), one
// warp per query head of the group.  Also lays the kept, scaled q' out as the
// B operands of the attend kernel's tensor-core tiles.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace dqk {

// Warp-wide bitonic sort, descending, of 32*E distinct 64-bit keys; element
// index lane*E + e.  Stages whose partner distance is below E stay in
// registers, the others exchange through shuffles.
template <int E>
__device__ __forceinline__ void warp_bitonic_desc(unsigned long long (&v)[E], int lane) {
    constexpr int N = 32 * E;
#pragma unroll
    for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
            if (jj >= E) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int i = lane * E + e;
                    const unsigned long long o = __shfl_xor_sync(0xffffffffu, v[e], jj / E);
                    const bool keep_max = ((i & jj) == 0) == ((i & k) == 0);
                    v[e] = keep_max ? (v[e] > o ? v[e] : o) : (v[e] < o ? v[e] : o);
                }
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int pe = e ^ jj;
                    if (pe > e) {
                        const int i = lane * E + e;
                        const unsigned long long a = v[e], b = v[pe];
                        const bool desc = (i & k) == 0;
                        if (desc ? (a < b) : (a > b)) {
                            v[e] = b;
                            v[pe] = a;
                        }
                    }
                }
            }
        }
    }
}

// Query fragments of one (sequence, kv head), consumed by k_attend:
//   qf  [B*Hkv][NT][NG][2][32] uint2   per lane: the f16x2 pairs (b0b1, b2b3)
//       of the QK B operand of k-step s of group g: rows = channels
//       32g+16s+2*tig+{0,1} (and +8), column n = gid -> query head 4*nt + gid/2,
//       gid even: fp16 high part, odd: low part of qs = q'_c * log2(e)/sqrt(d)
//       on kept channels c >= 1, 0 elsewhere.
//   qm  [B*Hkv][NT][32] uint32         per lane: rows 2*tig, 2*tig+1 of the
//       min-term B operand: Qsum_{g,h} = sum of qs over the group's kept
//       channels (hi/lo by column parity as above).
//   q0  [B][Hq] float                  qs of channel 0 (always kept).
template <int D>
struct QFrag {
    static constexpr int NG = D / 32;
};

__device__ __forceinline__ uint16_t f16_piece(float x, int piece) {
    const __half hi = __float2half_rn(x);
    if (piece == 0) return __half_as_ushort(hi);
    return __half_as_ushort(__float2half_rn(x - __half2float(hi)));
}

template <int D>
__global__ void __launch_bounds__(256) k_qprep(const float *__restrict__ t_q, const void *__restrict__ q,
                                              int dtype, int hq, int hkv, int pct, float qscale,
                                              uint2 *__restrict__ qf, uint32_t *__restrict__ qm,
                                              float *__restrict__ q0, int16_t *__restrict__ sel_out) {
    constexpr int NG = D / 32;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int G = hq / hkv;
    const int NT = G > 4 ? 2 : 1;
    float *tq = reinterpret_cast<float *>(smem_raw);                 // [D][D+1]
    float *qrow = tq + D * (D + 1);                                   // [G][D]  input, then qs
    float *qsum = qrow + G * D;                                       // [G][NG]
    unsigned char *mask = reinterpret_cast<unsigned char *>(qsum + G * NG);  // [G][D]
    const int j = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dependents_launch();   // the attend kernel may start streaming pages now
    const float *T = t_q + (size_t)j * D * D;
    for (int idx = threadIdx.x; idx < D * D; idx += blockDim.x) tq[(idx / D) * (D + 1) + (idx % D)] = T[idx];
    if (warp < G) {
        const size_t base = ((size_t)b * hq + j * G + warp) * D;
        for (int c = lane; c < D; c += 32) {
            qrow[warp * D + c] = (dtype == DQK_BF16) ? bf16_to_f32(reinterpret_cast<const uint16_t *>(q)[base + c])
                                                     : reinterpret_cast<const float *>(q)[base + c];
            mask[warp * D + c] = 0;
        }
    }
    __syncthreads();
    if (warp < G) {
        const int h = j * G + warp;
        const int nk = keep_count(D, pct);
        float qp[NG];
        unsigned long long key[NG];
#pragma unroll
        for (int m = 0; m < NG; ++m) {
            const int c = lane + 32 * m;
            const float *row = &tq[c * (D + 1)];
            double s = 0.0;
#pragma unroll 8
            for (int i = 0; i < D; ++i) s = fma((double)row[i], (double)qrow[warp * D + i], s);
            qp[m] = __double2float_rn(s);
            // descending |q'|, then ascending channel; channel 0 sorts last (key 0)
            key[m] = (c == 0) ? 0ull
                              : (((unsigned long long)(__float_as_uint(qp[m]) & 0x7fffffffu) << 32) |
                                 (unsigned long long)(0xffffffffu - (unsigned)c));
        }
        warp_bitonic_desc<NG>(key, lane);
#pragma unroll
        for (int e = 0; e < NG; ++e)
            if (lane * NG + e < nk - 1) mask[warp * D + (int)(0xffffffffu - (unsigned)(key[e] & 0xffffffffull))] = 1;
        if (lane == 0) mask[warp * D] = 1;
        __syncwarp();
        int written = 0;
#pragma unroll
        for (int m = 0; m < NG; ++m) {
            const int c = lane + 32 * m;
            const bool keep = mask[warp * D + c] != 0;
            const unsigned bal = __ballot_sync(0xffffffffu, keep);
            if (sel_out && keep)
                sel_out[((size_t)b * hq + h) * nk + written + __popc(bal & ((1u << lane) - 1u))] = (int16_t)c;
            written += __popc(bal);
            const float qs = qp[m] * qscale;
            if (c == 0) q0[(size_t)b * hq + h] = qs;
            const float v = (keep && c != 0) ? qs : 0.0f;
            qrow[warp * D + c] = v;
            // group sums of the kept, scaled channels (channel 0 excluded)
            float gs = v;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) gs += __shfl_xor_sync(0xffffffffu, gs, o);
            if (lane == 0) qsum[warp * NG + m] = gs;
        }
    }
    __syncthreads();
    // lay out the B-operand fragments
    const size_t bj = (size_t)b * hkv + j;
    for (int idx = threadIdx.x; idx < NT * NG * 2 * 32; idx += blockDim.x) {
        const int L = idx & 31, s = (idx >> 5) & 1, g = (idx >> 6) % NG, nt = (idx >> 6) / NG;
        const int gid = L >> 2, tig = L & 3, hl = 4 * nt + (gid >> 1), piece = gid & 1;
        const int c0 = 32 * g + 16 * s + 2 * tig;
        uint32_t w0 = 0, w1 = 0;
        if (hl < G) {
            const float *r = &qrow[hl * D];
            w0 = (uint32_t)f16_piece(r[c0], piece) | ((uint32_t)f16_piece(r[c0 + 1], piece) << 16);
            w1 = (uint32_t)f16_piece(r[c0 + 8], piece) | ((uint32_t)f16_piece(r[c0 + 9], piece) << 16);
        }
        qf[(((bj * NT + nt) * NG + g) * 2 + s) * 32 + L] = make_uint2(w0, w1);
    }
    for (int idx = threadIdx.x; idx < NT * 32; idx += blockDim.x) {
        const int L = idx & 31, nt = idx >> 5;
        const int gid = L >> 2, tig = L & 3, hl = 4 * nt + (gid >> 1), piece = gid & 1;
        uint32_t w = 0;
        if (hl < G) {
            const int g0 = 2 * tig, g1 = 2 * tig + 1;
            const uint32_t lo = g0 < NG ? f16_piece(qsum[hl * NG + g0], piece) : 0u;
            const uint32_t hi = g1 < NG ? f16_piece(qsum[hl * NG + g1], piece) : 0u;
            w = lo | (hi << 16);
        }
        qm[(bj * NT + nt) * 32 + L] = w;
    }
}

}  // namespace dqk
