// common.cuh -- shared pieces of libdualqk's kernels: the paged block layout,
// IEEE rounding helpers, and the device error word.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/dualqk.h"

namespace dqk {

constexpr int kPage = 16;   // tokens per page
constexpr int kGroup = 32;  // channels per quantization group

// Error bits OR-ed into the device error word.
constexpr unsigned kErrBounds = 1u;
constexpr unsigned kErrTimeout = 2u;

// Byte offsets of the sections of one (page, kv head) block; see dualqk.h.
// ns = scale groups per token: d / 32, or 1 (one group over the whole head).
struct Layout {
    int d, ns, kc, ks, km, k0, vc, vs, vm, v0, bytes;
};

__host__ __device__ constexpr Layout make_layout(int d, int v_ch0, int ns) {
    Layout L{};
    L.d = d;
    L.ns = ns;
    L.kc = 0;
    L.ks = 4 * d;
    L.km = L.ks + 32 * ns;
    L.k0 = L.km + 32 * ns;
    L.vc = L.k0 + 32;
    L.vs = L.vc + 4 * d;
    L.vm = L.vs + 32 * ns;
    L.v0 = L.vm + 32 * ns;
    L.bytes = L.v0 + (v_ch0 ? 32 : 0);
    return L;
}

// Key code of (token t, channel c): byte offset of its 32-bit word inside the
// K code section and the bit of its 2-bit field.  The order is the u8 A
// operand of m16n8k32 tiles with tokens as rows and the 32 channels of one
// group as columns: register r (row t%8 + 8*(r&1), columns 16*(r>>1) +
// 4*(lane%4) + byte) of group g sits in field g (NG = 4) of that byte, so one
// AND with 0x03030303 << 2g yields the operand with values code * 4^g.  With
// NG = 2 the registers r >= 2 take fields 2 and 3 of the words of r - 2.
__host__ __device__ __forceinline__ void kcode_pos(int ng, int t, int c, int &word_off, int &bit) {
    const int g = c >> 5, cc = c & 31;
    const int r = 2 * (cc >> 4) + (t >> 3);
    const int lane = 4 * (t & 7) + ((cc & 15) >> 2);
    const int j = cc & 3;
    const int W = r % ng, f = g + ng * (r / ng);
    word_off = (lane * ng + W) * 4;
    bit = 8 * j + 2 * f;
}

// Value code of (token t, channel c): the A operand of an m16n8k16 tile with
// channels as rows and tokens as columns (O^T = V^T P).  NG = 4: register k of
// m-tile m (rows 16m + gid + 8*(k&1), columns 2*tig + 8*(k>>1) + e) is word k
// of the lane, field m of half e, so each m-tile reads one field position of
// all four words (one AND each, no shift for fields 0..4).  NG = 2: the
// m-tiles' registers follow each other through the fields of the two words.
__host__ __device__ __forceinline__ void vcode_pos(int ng, int t, int c, int &word_off, int &bit) {
    const int m = c >> 4, r = c & 15, cr = r >> 3, gid = r & 7;
    const int tb = t >> 3, tig = (t & 7) >> 1, e = t & 1;
    const int lane = gid * 4 + tig;
    if (ng == 4) {
        word_off = (lane * 4 + cr + 2 * tb) * 4;
        bit = e * 16 + 2 * m;
        return;
    }
    const int q = (m * 2 + cr) * 2 + tb;
    word_off = (lane * ng + (q >> 3)) * 4;
    bit = e * 16 + 2 * (q & 7);
}

__host__ __device__ __forceinline__ int kscale_idx(int ng, int t, int g) { return t * ng + g; }
__host__ __device__ __forceinline__ int k0_idx(int t) { return 2 * (t & 7) + (t >> 3); }
__host__ __device__ __forceinline__ int vscale_idx(int ng, int t, int g) {
    return 2 * (ng * (t >> 1) + g) + (t & 1);
}

// n_keep = d - floor(pct*d/100): channel 0 is always kept and counted.
__host__ __device__ __forceinline__ int keep_count(int d, int pct) { return d - (pct * d) / 100; }

// ---------------------------------------------------------------------------
// IEEE 754 rounding, from the format definitions (bit arithmetic only).
// ---------------------------------------------------------------------------

// binary64 -> binary16, round to nearest even, |x| >= 65504 saturates to the
// largest finite value, NaN -> 0x7E00.
__device__ __forceinline__ uint16_t f64_to_f16_rne(double x) {
    unsigned long long b = (unsigned long long)__double_as_longlong(x);
    uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
    unsigned long long a = b & 0x7FFFFFFFFFFFFFFFull;
    if (a > 0x7FF0000000000000ull) return 0x7E00u;
    if (__longlong_as_double((long long)a) >= 65504.0) return (uint16_t)(sign | 0x7BFFu);
    int e = (int)(a >> 52) - 1023;
    if (e < -25) return sign;  // below half the smallest subnormal (or a double subnormal)
    unsigned long long m = (a & 0x000FFFFFFFFFFFFFull) | 0x0010000000000000ull;  // 53 bits
    int shift = (e >= -14) ? 42 : (28 - e);  // keep 11 bits (normal) or units of 2^-24
    unsigned long long q = m >> shift;
    unsigned long long rem = m & ((1ull << shift) - 1ull);
    unsigned long long half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (q & 1ull))) ++q;
    if (e >= -14) {
        int be = e + 15;
        if (q == 2048ull) { q = 1024ull; ++be; }
        if (be >= 31) return (uint16_t)(sign | 0x7BFFu);
        return (uint16_t)(sign | (uint16_t)(be << 10) | (uint16_t)(q - 1024ull));
    }
    return (uint16_t)(sign | (uint16_t)q);  // q == 1024 encodes the smallest normal
}

__device__ __forceinline__ double f16_to_f64(uint16_t h) {
    return (double)__half2float(__ushort_as_half(h));  // exact widening
}

// binary32 -> bfloat16, round to nearest even (NaN -> quiet NaN).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float x) {
    uint32_t u = __float_as_uint(x);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0x7FC0u;
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

}  // namespace dqk

// One error word per device, OR-ed by kernels, read by dqk_last_device_error.
// (libdualqk is a single translation unit: dualqk.cu includes every kernel.)
__device__ unsigned int g_dqk_device_error = 0;

__device__ __forceinline__ void dqk_flag_error(unsigned bits) { atomicOr(&g_dqk_device_error, bits); }
