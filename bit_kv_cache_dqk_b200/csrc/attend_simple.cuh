// attend_simple.cuh -- first split-K attend kernel over the INT2 cache on CUDA
// cores (one CTA per (split, kv head, sequence)); the LSE combine.
#pragma once

#include "common.cuh"

namespace dqk {

constexpr int kSimplePagesPerSplit = 32;  // 512 tokens per split
constexpr int kSimpleThreads = 128;

__device__ __forceinline__ uint32_t ld_word(const uint8_t *blk, int off) {
    return *reinterpret_cast<const uint32_t *>(blk + off);
}
__device__ __forceinline__ float ld_half(const uint8_t *blk, int off_bytes) {
    return __half2float(*reinterpret_cast<const __half *>(blk + off_bytes));
}

// Partials: part_o [B][Hq][NS][D] (sum_t p_t v_t with p_t = exp(s_t - m)),
// part_ml [B][Hq][NS][2] = (m, l).  Scores in natural-log units.
template <int D, int G>
__global__ void __launch_bounds__(kSimpleThreads) k_attend_simple(
    const uint8_t *__restrict__ pool, int hkv, int v_ch0, long long num_pages,
    const int *__restrict__ seq_lens, const int *__restrict__ page_table, int max_pages,
    const float *__restrict__ qsel, int ns, float *__restrict__ part_o, float *__restrict__ part_ml) {
    constexpr int NG = D / 32;
    constexpr int TS = kSimplePagesPerSplit * kPage;
    __shared__ float qs[G][D];
    __shared__ float sc[TS][G];
    __shared__ float red[kSimpleThreads / 32][G];
    __shared__ float mrow[G], lrow[G];
    const int sp = blockIdx.x, j = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int hq = hkv * G;
    const int Lb = seq_lens[b];
    const int t0 = sp * TS;
    if (t0 >= Lb) return;
    const int t1 = min(Lb, t0 + TS);
    const Layout L = make_layout(D, v_ch0);
    for (int idx = tid; idx < G * D; idx += blockDim.x)
        qs[idx / D][idx % D] = qsel[((size_t)b * hq + j * G + idx / D) * D + idx % D];
    __syncthreads();
    const float inv_sqrt_d = 1.0f / sqrtf((float)D);
    for (int t = t0 + tid; t < t1; t += blockDim.x) {
        const int page = t / kPage, slot = t % kPage;
        const int phys = page < max_pages ? page_table[(size_t)b * max_pages + page] : -1;
        float acc[G];
        if (phys < 0 || phys >= num_pages) {
            dqk_flag_error(kErrBounds);
#pragma unroll
            for (int h = 0; h < G; ++h) sc[t - t0][h] = -INFINITY;
            continue;
        }
        const uint8_t *blk = pool + ((size_t)phys * hkv + j) * L.bytes;
        const float k0 = bf16_to_f32(*reinterpret_cast<const uint16_t *>(blk + L.k0 + 2 * k0_idx(slot)));
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = qs[h][0] * k0;
        for (int g = 0; g < NG; ++g) {
            const float s = ld_half(blk, L.ks + 2 * kscale_idx(NG, slot, g));
            const float mn = ld_half(blk, L.km + 2 * kscale_idx(NG, slot, g));
            for (int cc = (g == 0 ? 1 : 0); cc < 32; ++cc) {
                const int c = g * 32 + cc;
                int off, bit;
                kcode_pos(NG, slot, c, off, bit);
                const float kv = mn + (float)((ld_word(blk, L.kc + off) >> bit) & 3u) * s;
#pragma unroll
                for (int h = 0; h < G; ++h) acc[h] = fmaf(qs[h][c], kv, acc[h]);
            }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) sc[t - t0][h] = acc[h] * inv_sqrt_d;
    }
    __syncthreads();
    // per-head max and sum
    for (int h = 0; h < G; ++h) {
        float mx = -INFINITY;
        for (int t = tid; t < t1 - t0; t += blockDim.x) mx = fmaxf(mx, sc[t][h]);
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if ((tid & 31) == 0) red[tid >> 5][h] = mx;
    }
    __syncthreads();
    if (tid < G) {
        float mx = -INFINITY;
        for (int w = 0; w < kSimpleThreads / 32; ++w) mx = fmaxf(mx, red[w][tid]);
        mrow[tid] = mx;
    }
    __syncthreads();
    for (int h = 0; h < G; ++h) {
        float l = 0.0f;
        for (int t = tid; t < t1 - t0; t += blockDim.x) {
            const float p = (mrow[h] == -INFINITY) ? 0.0f : __expf(sc[t][h] - mrow[h]);
            sc[t][h] = p;
            l += p;
        }
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        __syncthreads();
        if ((tid & 31) == 0) red[tid >> 5][h] = l;
        __syncthreads();
    }
    if (tid < G) {
        float l = 0.0f;
        for (int w = 0; w < kSimpleThreads / 32; ++w) l += red[w][tid];
        lrow[tid] = l;
    }
    __syncthreads();
    for (int c = tid; c < D; c += blockDim.x) {
        float o[G];
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] = 0.0f;
        const int g = c / 32;
        for (int t = t0; t < t1; ++t) {
            const int page = t / kPage, slot = t % kPage;
            const int phys = page < max_pages ? page_table[(size_t)b * max_pages + page] : -1;
            if (phys < 0 || phys >= num_pages) continue;
            const uint8_t *blk = pool + ((size_t)phys * hkv + j) * L.bytes;
            float vv;
            if (c == 0 && v_ch0) {
                vv = bf16_to_f32(*reinterpret_cast<const uint16_t *>(blk + L.v0 + 2 * slot));
            } else {
                int off, bit;
                vcode_pos(NG, slot, c, off, bit);
                const float s = ld_half(blk, L.vs + 2 * vscale_idx(NG, slot, g));
                const float mn = ld_half(blk, L.vm + 2 * vscale_idx(NG, slot, g));
                vv = mn + (float)((ld_word(blk, L.vc + off) >> bit) & 3u) * s;
            }
#pragma unroll
            for (int h = 0; h < G; ++h) o[h] = fmaf(sc[t - t0][h], vv, o[h]);
        }
#pragma unroll
        for (int h = 0; h < G; ++h)
            part_o[(((size_t)b * hq + j * G + h) * ns + sp) * D + c] = o[h];
    }
    if (tid < G) {
        const size_t i = ((size_t)b * hq + j * G + tid) * ns + sp;
        part_ml[2 * i] = mrow[tid];
        part_ml[2 * i + 1] = lrow[tid];
    }
}

// out[b][h] = sum_s o_s e^{m_s - m*} / sum_s l_s e^{m_s - m*}; zero when L_b == 0.
template <int D>
__global__ void k_combine_simple(const int *__restrict__ seq_lens, int hq, int ns, int tokens_per_split,
                                 const float *__restrict__ part_o, const float *__restrict__ part_ml,
                                 float *__restrict__ out) {
    const int h = blockIdx.x, b = blockIdx.y;
    const int Lb = seq_lens[b];
    const int n = Lb > 0 ? min(ns, (Lb + tokens_per_split - 1) / tokens_per_split) : 0;
    const size_t row = (size_t)b * hq + h;
    float mstar = -INFINITY;
    for (int s = 0; s < n; ++s) mstar = fmaxf(mstar, part_ml[2 * (row * ns + s)]);
    float den = 0.0f;
    for (int s = 0; s < n; ++s) {
        const float m = part_ml[2 * (row * ns + s)];
        if (m != -INFINITY) den += part_ml[2 * (row * ns + s) + 1] * __expf(m - mstar);
    }
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        float num = 0.0f;
        for (int s = 0; s < n; ++s) {
            const float m = part_ml[2 * (row * ns + s)];
            if (m != -INFINITY) num += part_o[(row * ns + s) * D + c] * __expf(m - mstar);
        }
        out[row * D + c] = (den > 0.0f) ? num / den : 0.0f;
    }
}

}  // namespace dqk
