// qprep.cuh -- k_qprep: query transform q' = T_Q q and dynamic channel
// selection (keep channel 0 and the largest-|q'| channels; "Why the cache
// becomes a bottleneck": query-channel pruning; "Throughput on SGLang": 40 %
// of key channels removed from reads).  One CTA per (sequence, kv head), one
// warp per query head of the group.
#pragma once

#include "common.cuh"

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

// Outputs per (b, h):
//   qsel   fp32 [B][Hq][D]  q'_c on kept channels, 0 elsewhere (channel 0 kept)
//   sel    int16 [B][Hq][n_keep] kept channels ascending (nullable)
template <int D>
__global__ void __launch_bounds__(256) k_qprep(const float *__restrict__ t_q, const void *__restrict__ q,
                                              int dtype, int hq, int hkv, int pct,
                                              float *__restrict__ qsel, int16_t *__restrict__ sel_out) {
    constexpr int NG = D / 32;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *tq = reinterpret_cast<float *>(smem_raw);            // [D][D+1]
    float *qrow = tq + D * (D + 1);                              // [G][D]
    unsigned char *mask = reinterpret_cast<unsigned char *>(qrow + (hq / hkv) * D);  // [G][D]
    const int j = blockIdx.x, b = blockIdx.y, G = hq / hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *T = t_q + (size_t)j * D * D;
    for (int idx = threadIdx.x; idx < D * D; idx += blockDim.x) tq[(idx / D) * (D + 1) + (idx % D)] = T[idx];
    if (warp < G) {
        const int h = j * G + warp;
        const size_t base = ((size_t)b * hq + h) * D;
        for (int c = lane; c < D; c += 32) {
            qrow[warp * D + c] = (dtype == DQK_BF16) ? bf16_to_f32(reinterpret_cast<const uint16_t *>(q)[base + c])
                                                     : reinterpret_cast<const float *>(q)[base + c];
            mask[warp * D + c] = 0;
        }
    }
    __syncthreads();
    if (warp >= G) return;
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
        // descending |q'| then ascending channel; channel 0 sorts last (key 0)
        key[m] = (c == 0) ? 0ull
                          : (((unsigned long long)(__float_as_uint(qp[m]) & 0x7fffffffu) << 32) |
                             (unsigned long long)(0xffffffffu - (unsigned)c));
    }
    // NG keys per lane; the sort wants them at index lane*NG + e.
    warp_bitonic_desc<NG>(key, lane);
#pragma unroll
    for (int e = 0; e < NG; ++e) {
        const int rank = lane * NG + e;
        if (rank < nk - 1) mask[warp * D + (int)(0xffffffffu - (unsigned)(key[e] & 0xffffffffull))] = 1;
    }
    if (lane == 0) mask[warp * D] = 1;
    __syncwarp();
    const size_t base = ((size_t)blockIdx.y * hq + h) * D;
    int written = 0;
#pragma unroll
    for (int m = 0; m < NG; ++m) {
        const int c = lane + 32 * m;
        const bool keep = mask[warp * D + c] != 0;
        qsel[base + c] = keep ? qp[m] : 0.0f;
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (sel_out && keep)
            sel_out[((size_t)blockIdx.y * hq + h) * nk + written + __popc(bal & ((1u << lane) - 1u))] = (int16_t)c;
        written += __popc(bal);
    }
}

}  // namespace dqk
