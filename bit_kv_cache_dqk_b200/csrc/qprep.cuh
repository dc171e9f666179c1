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

// Query fragments of one (sequence, kv head), consumed by k_attend, with
// qs = q'_c * log2(e)/sqrt(d) on kept channels c >= 1 (0 elsewhere):
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
__device__ __forceinline__ uint16_t f16_piece(float x, int piece) {
    const __half hi = __float2half_rn(x);
    if (piece == 0) return __half_as_ushort(hi);
    return __half_as_ushort(__float2half_rn(x - __half2float(hi)));
}

constexpr int kQprepThreads = 512;

// Shared memory of k_qprep: T_Q[j] in fp32 with rows padded to D+4 floats
// (conflict-free 16-byte row reads), the query rows in fp64, per-head sort
// buffers and the outputs before they are laid out.  (T_Q held in fp64 would
// double this; the larger CTAs then slow a co-running append.)
__host__ __device__ constexpr size_t qprep_smem_bytes(int D, int G) {
    return (size_t)D * (D + 4) * 4 + (size_t)G * D * 8 + (size_t)kQprepThreads * 8 + (size_t)G * (D / 32) * 8 +
           (size_t)G * (D / 32 + 1) * 4 + (size_t)G * D * 3 + 64;
}

// One thread per (query head, channel), kQprepThreads / D heads per pass.
// Launched with programmatic stream serialization: it reads its inputs and
// computes q' and the selection while an earlier append may still be running,
// waits for the earlier work before writing anything, then releases the
// attend kernel.
template <int D>
__global__ void __launch_bounds__(kQprepThreads) k_qprep(const float *__restrict__ t_q, const void *__restrict__ q,
                                                        int dtype, int hq, int hkv, int pct, float qscale,
                                                        uint2 *__restrict__ qf, float *__restrict__ qk,
                                                        uint32_t *__restrict__ qm, float *__restrict__ q0,
                                                        int16_t *__restrict__ sel_out, int write_first) {
    constexpr int NG = D / 32;
    constexpr int kRow = D + 4;                       // padded fp32 row of T_Q
    constexpr int kHeadsPerPass = kQprepThreads / D;
    constexpr int kWarpsPerHead = D / 32;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int G = hq / hkv;
    const int NT = G > 4 ? 2 : 1;
    float *tq = reinterpret_cast<float *>(smem_raw);                                  // [D][D+4]
    double *qin = reinterpret_cast<double *>(tq + D * kRow);                         // [G][D]
    unsigned long long *xbuf = reinterpret_cast<unsigned long long *>(qin + G * D);  // [threads] sort exchange
    float *qsum = reinterpret_cast<float *>(xbuf + kQprepThreads);                   // [G][NG]
    float *sig = qsum + G * NG;                                                       // [G][NG]  p_g
    float *gmax = sig + G * NG;                                                       // [G][NG]  largest |qs|
    float *shd = gmax + G * NG;                                                       // [G]      sigma_h
    signed char *q8 = reinterpret_cast<signed char *>(shd + G);                      // [G][2][D] pieces
    unsigned char *mask = reinterpret_cast<unsigned char *>(q8 + G * 2 * D);         // [G][D]
    int *wcount = reinterpret_cast<int *>(mask + G * D + ((16 - (G * D) % 16) % 16)); // [threads/32] kept per warp
    const int j = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = threadIdx.x % D, hp = threadIdx.x / D;   // channel, head slot of the pass
    const int nk = keep_count(D, pct);

    {   // stage T_Q[j] (fp32, padded rows) and the query rows (fp64)
        constexpr int n4 = D * D / 4, kIn = (n4 + kQprepThreads - 1) / kQprepThreads;
        const float4 *src = reinterpret_cast<const float4 *>(t_q + (size_t)j * D * D);
        float4 v[kIn];
#pragma unroll
        for (int u = 0; u < kIn; ++u) {
            const int i4 = threadIdx.x + u * kQprepThreads;
            if (i4 < n4) v[u] = src[i4];
        }
        const size_t qbase = ((size_t)b * hq + (size_t)j * G) * D;
        for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x)
            qin[idx] = (double)((dtype == DQK_BF16) ? bf16_to_f32(reinterpret_cast<const uint16_t *>(q)[qbase + idx])
                                                    : reinterpret_cast<const float *>(q)[qbase + idx]);
#pragma unroll
        for (int u = 0; u < kIn; ++u) {
            const int i4 = threadIdx.x + u * kQprepThreads;
            if (i4 < n4) {
                const int e = 4 * i4, row = e / D, col = e % D;
                *reinterpret_cast<float4 *>(&tq[row * kRow + col]) = v[u];
            }
        }
    }
    __syncthreads();

    // write_first: the kernel before this one on the stream (a cache append
    // launched without programmatic serialization) writes nothing this kernel
    // reads or writes, and everything before it has finished, so the outputs
    // are written at once and the wait for it comes last (this kernel's
    // completion then implies the append's).  Otherwise the outputs wait for
    // every earlier kernel of the stream.
    bool waited = write_first != 0;
    for (int h0 = 0; h0 < G; h0 += kHeadsPerPass) {
        const int hl = h0 + hp;                 // local query head of this thread
        const bool active = hl < G;
        const int h = j * G + hl;
        // q'_c = sum_i T_Q[c][i] q_i, ascending i, exact fp32 x fp32 products
        // accumulated in fp64, rounded once to fp32
        float qp = 0.0f;
        if (active) {
            const float *row = &tq[c * kRow];
            const double *x = &qin[hl * D];
            double acc = 0.0;
#pragma unroll
            for (int i = 0; i < D; i += 4) {
                const float4 t4 = *reinterpret_cast<const float4 *>(&row[i]);
                acc = fma((double)t4.x, x[i + 0], acc);
                acc = fma((double)t4.y, x[i + 1], acc);
                acc = fma((double)t4.z, x[i + 2], acc);
                acc = fma((double)t4.w, x[i + 3], acc);
            }
            qp = __double2float_rn(acc);
        }
        // selection: bitonic sort (descending) of the head's D keys, one per
        // thread: |q'| bits, then ascending channel; channel 0 sorts last
        unsigned long long key = (c == 0) ? 0ull
                                          : (((unsigned long long)(__float_as_uint(qp) & 0x7fffffffu) << 32) |
                                             (unsigned long long)(0xffffffffu - (unsigned)c));
#pragma unroll
        for (int k = 2; k <= D; k <<= 1) {
#pragma unroll
            for (int jj = k >> 1; jj > 0; jj >>= 1) {
                unsigned long long o;
                if (jj < 32) {
                    o = __shfl_xor_sync(0xffffffffu, key, jj);
                } else {
                    xbuf[threadIdx.x] = key;
                    __syncthreads();
                    o = xbuf[threadIdx.x ^ jj];
                    __syncthreads();
                }
                const bool keep_max = ((c & jj) == 0) == ((c & k) == 0);
                key = keep_max ? (key > o ? key : o) : (key < o ? key : o);
            }
        }
        // position c of the sorted order holds the c-th largest key
        if (active) mask[hl * D + c] = 0;
        __syncthreads();
        if (active && c < nk - 1) mask[hl * D + (int)(0xffffffffu - (unsigned)(key & 0xffffffffull))] = 1;
        if (active && c == 0) mask[hl * D] = 1;
        __syncthreads();
        const bool keep = active && mask[hl * D + c] != 0;
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) wcount[warp] = __popc(bal);
        // scaled q' on kept channels >= 1; group sums and two int8 pieces
        // (warp = one group of one head) relative to sigma_g = sigma_h * 2^-e,
        // the smallest such value not below the group's largest |qs| / 127, so
        // that sigma_g / sigma_h is a power of two
        const float qs = qp * qscale;
        const float v = (keep && c != 0) ? qs : 0.0f;
        float gs = v, gm = fabsf(v);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            gs += __shfl_xor_sync(0xffffffffu, gs, o);
            gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
        }
        const int g = c >> 5;
        if (active && lane == 0) gmax[hl * NG + g] = gm;
        __syncthreads();
        float hm = 0.0f;
        if (active)
            for (int gg = 0; gg < NG; ++gg) hm = fmaxf(hm, gmax[hl * NG + gg]);
        const float sh = hm / 127.0f, tg = gm / 127.0f;
        int e = 0;
        if (tg > 0.0f) {
            e = ilogbf(sh) - ilogbf(tg);   // >= 0: sh >= tg
            if (ldexpf(sh, -e) < tg) --e;
        }
        const float sgm = ldexpf(sh, -e);   // in [tg, 2 tg)
        int q1 = 0, q2 = 0;
        if (sgm > 0.0f) {
            const float x = v / sgm;
            q1 = max(-127, min(127, __float2int_rn(x)));
            q2 = max(-128, min(127, __float2int_rn((x - (float)q1) * 256.0f)));
        }
        if (active) {
            q8[(hl * 2 + 0) * D + c] = (signed char)q1;
            q8[(hl * 2 + 1) * D + c] = (signed char)q2;
            if (lane == 0) {
                qsum[hl * NG + g] = gs;
                sig[hl * NG + g] = ldexpf(1.0f, -e - 2 * g);
            }
            if (c == 0) shd[hl] = sh;
        }
        __syncthreads();
        if (!waited) {
            grid_dependency_wait();     // earlier work on the stream (e.g. a cache append) is complete
            grid_dependents_launch();   // the attend kernel may start streaming pages now
            waited = true;
        }
        if (active) {
            // kept channels before c: earlier warps of this head, then lanes below
            int before = __popc(bal & ((1u << lane) - 1u));
            for (int w = warp - (warp % kWarpsPerHead); w < warp; ++w) before += wcount[w];
            if (sel_out && keep) sel_out[((size_t)b * hq + h) * nk + before] = (int16_t)c;
            if (c == 0) q0[(size_t)b * hq + h] = qs;
        }
        __syncthreads();
    }
    // lay out the B-operand fragments
    const size_t bj = (size_t)b * hkv + j;
    for (int idx = threadIdx.x; idx < NT * NG * 32; idx += blockDim.x) {
        const int L = idx & 31, g = (idx >> 5) % NG, nt = (idx >> 5) / NG;
        const int gid = L >> 2, tig = L & 3, hl = 4 * nt + (gid >> 1), piece = gid & 1;
        uint32_t w0 = 0, w1 = 0;
        if (hl < G) {
            const unsigned char *r = reinterpret_cast<const unsigned char *>(&q8[(hl * 2 + piece) * D + 32 * g]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                w0 |= (uint32_t)r[4 * tig + i] << (8 * i);
                w1 |= (uint32_t)r[16 + 4 * tig + i] << (8 * i);
            }
        }
        qf[((bj * NT + nt) * NG + g) * 32 + L] = make_uint2(w0, w1);
    }
    for (int idx = threadIdx.x; idx < NT * (NG + 1) * 4; idx += blockDim.x) {
        const int hh = idx & 3, g = (idx >> 2) % (NG + 1), nt = (idx >> 2) / (NG + 1), hl = 4 * nt + hh;
        qk[((bj * NT + nt) * (NG + 1) + g) * 4 + hh] = hl < G ? (g < NG ? sig[hl * NG + g] : shd[hl]) : 0.0f;
    }
    for (int idx = threadIdx.x; idx < NT * 32; idx += blockDim.x) {
        const int L = idx & 31, nt = idx >> 5;
        const int gid = L >> 2, tig = L & 3, hl = 4 * nt + (gid >> 1);
        uint32_t w = 0;
        if (hl < G && (gid & 1) == 0) {
            // rows k = 2*tig, 2*tig + 1: piece k / NG (0 high, 1 low) of group k % NG
            const int k0 = 2 * tig, k1 = 2 * tig + 1;
            const uint32_t r0 = k0 < 2 * NG ? f16_piece(qsum[hl * NG + k0 % NG], k0 / NG) : 0u;
            const uint32_t r1 = k1 < 2 * NG ? f16_piece(qsum[hl * NG + k1 % NG], k1 / NG) : 0u;
            w = r0 | (r1 << 16);
        }
        qm[(bj * NT + nt) * 32 + L] = w;
    }
    if (write_first) {
        grid_dependency_wait();     // the append is complete
        grid_dependents_launch();   // the attend kernel may start streaming pages now
    }
}

}  // namespace dqk
