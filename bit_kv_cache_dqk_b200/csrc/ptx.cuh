// ptx.cuh -- thin inline-PTX wrappers used by the attend kernel: mbarriers,
// 1-D bulk async copies (TMA engine), tensor-core MMA, bit tricks.
#pragma once

#include <stdint.h>

namespace dqk {

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that may suspend the thread for up to `hint_ns` before returning.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Wait for the phase of `parity` to complete, giving up after `limit_ns`.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t limit_ns,
                                                  uint32_t hint_ns = 0) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (hint_ns ? mbar_try_wait_hint(bar, parity, hint_ns) : mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0 && global_timer_ns() - t0 > limit_ns) return false;
    }
}

// 16-byte load of read-only global data through the non-coherent path, as an
// asm statement: the front end issues it where it stands; how many such loads
// the code generator keeps in flight depends on the registers it allots.
__device__ __forceinline__ float4 ld_nc_f4(const float4 *ptr) {
    float4 v;
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(ptr));
    return v;
}

// 16-byte asynchronous copy global -> shared (L2 only; both addresses 16-byte
// aligned); cp_async_wait_all waits for it.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// Scalar global loads as asm statements (issued where they stand, see above).
__device__ __forceinline__ float ld_f32_vol(const float *ptr) {
    float v;
    asm volatile("ld.global.f32 %0, [%1];" : "=f"(v) : "l"(ptr));
    return v;
}
__device__ __forceinline__ uint32_t ld_u16_vol(const uint16_t *ptr) {
    uint16_t v;
    asm volatile("ld.global.u16 %0, [%1];" : "=h"(v) : "l"(ptr));
    return v;
}

// Named barrier `id` over `n` threads: arrive without waiting, or arrive and
// wait.  (Barrier 0 is __syncthreads.)
__device__ __forceinline__ void named_bar_arrive(int id, int n) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// L2 policy for data read once per launch: evicted first, so the small
// tensors a decode step re-reads (page table, lengths, transforms, query
// fragments, split records) stay resident across steps.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// 1-D bulk copy global -> shared, completion counted on `bar` (no multicast).
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// The same with an L2 cache policy.
__device__ __forceinline__ void bulk_copy_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                                   uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Wait for all of this thread's cp.async copies in flight.
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Stage a row-major [n][n] fp32 matrix into shared memory as fp64 (exact),
// rows padded to n+1 doubles, so the sequential fp64 dot products read their
// operands without per-use conversions.  n must be a multiple of 4.
template <int n>
__device__ __forceinline__ void stage_f64_padded(double *dst, const float *src) {
    constexpr int kInFlight = 8;   // float4 loads a thread issues before converting
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    constexpr int n4 = n * n / 4;
    for (int base = threadIdx.x; base < n4; base += kInFlight * blockDim.x) {
        float4 v[kInFlight];
#pragma unroll
        for (int u = 0; u < kInFlight; ++u)
            if (base + u * blockDim.x < n4) v[u] = s4[base + u * blockDim.x];
#pragma unroll
        for (int u = 0; u < kInFlight; ++u) {
            const int idx4 = base + u * blockDim.x;
            if (idx4 < n4) {
                const int e = idx4 * 4, row = e / n, col = e % n;
                double *d = dst + row * (n + 1) + col;
                d[0] = (double)v[u].x;
                d[1] = (double)v[u].y;
                d[2] = (double)v[u].z;
                d[3] = (double)v[u].w;
            }
        }
    }
}

// Generic-proxy accesses made before these fences are ordered before the
// async-proxy (bulk copy) accesses issued after them: shared memory of this
// CTA, and global memory.
__device__ __forceinline__ void fence_proxy_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Address of the grid-wide barrier word that the driver sets up for a
// cooperative launch (the word cooperative groups' grid sync uses): the grid
// workspace { size, barrier } sits at the address held in environment
// registers 1 (high half) and 2 (low half).  Null when the launch was not
// cooperative.
__device__ __forceinline__ unsigned int *coop_barrier_word() {
    unsigned int hi, lo;
    asm volatile("mov.u32 %0, %%envreg1;" : "=r"(hi));
    asm volatile("mov.u32 %0, %%envreg2;" : "=r"(lo));
    const unsigned long long ws = ((unsigned long long)hi << 32) | lo;
    return ws ? reinterpret_cast<unsigned int *>(ws + 4) : nullptr;
}

// Grid barrier, called by one thread of every CTA.  CTA 0 adds 2^31 - (C - 1),
// the others add 1: the top bit of the word flips when the last CTA arrives
// and the low bits return to their value, so the word needs no reset between
// barriers or launches as long as every CTA arrives once at each of them.  The
// release add publishes what the CTA wrote before (and, through the CTA
// barrier that precedes the call, what its other threads wrote); the acquire
// polls make the other CTAs' writes visible.  Gives up after limit_ns (false).
__device__ __forceinline__ bool grid_sync_bounded(unsigned int *word, uint64_t limit_ns) {
    const unsigned int add = blockIdx.x == 0 ? 0x80000000u - (gridDim.x - 1u) : 1u;
    unsigned int old;
    asm volatile("atom.release.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(word), "r"(add) : "memory");
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if ((old ^ ld_acquire_gpu(word)) & 0x80000000u) return true;
        if (it >= 64u) {
            if ((it & 31u) == 0u && global_timer_ns() - t0 > limit_ns) return false;
            __nanosleep(40);
        }
    }
}

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// D += A * B, m16n8k16, fp16 operands, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Packed fp32 pairs (two IEEE operations in one instruction, sm_100):
// d = a * b + c, a + b and a * b lane by lane, each lane rounded as the scalar operation.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// D += A * B in place, m16n8k32, u8 x s8 operands, s32 accumulate.
__device__ __forceinline__ void mma_u8s8_acc(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}


// Two 2-bit codes at bit 2P of each 16-bit half of x -> an f16x2 holding the
// exact values 0..3.  OR-ing the field into the mantissa of 2^(10-2P) gives
// 2^(10-2P) + code (the field's weight equals one ulp there); subtracting
// 2^(10-2P) leaves the code.  P in 0..4.
template <int P>
__device__ __forceinline__ uint32_t codes_to_f16x2(uint32_t x) {
    static_assert(P >= 0 && P <= 4, "field position");
    constexpr uint32_t mask = (3u << (2 * P)) | (3u << (16 + 2 * P));
    constexpr uint32_t magic = ((25u - 2u * P) << 10) * 0x10001u;
    uint32_t v, r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(v) : "r"(x), "n"(mask), "r"(magic));
    asm("sub.f16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(magic));
    return r;
}

// Field i (0..7) of a code word: fields 0..4 in place, 5..7 from x >> 10.
template <int I>
__device__ __forceinline__ uint32_t code_field(uint32_t x, uint32_t x_hi) {
    if constexpr (I <= 4) return codes_to_f16x2<I>(x);
    else return codes_to_f16x2<I - 5>(x_hi);
}

// m16n8k16 with bf16 operands, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 8x8 b16 matrices from shared memory (lane L gives the row address of
// matrix L/8), plain or transposed.
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// 2^x, MUFU approximation (relative error ~2^-22); -inf -> 0.
__device__ __forceinline__ float fast_exp2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// fp16 halves of a word as fp32 (exact; one conversion each)
__device__ __forceinline__ float f16lo_to_f32(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu))); }
__device__ __forceinline__ float f16hi_to_f32(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }

// Shared-memory loads by 32-bit shared-window address.  volatile keeps them
// after the mbarrier wait that makes the stage's bytes visible.
__device__ __forceinline__ uint4 ld_s128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 ld_s64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t ld_s32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t ld_s16(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t ld_s8(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ void st_s32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v));
}
__device__ __forceinline__ void st_s64(uint32_t a, uint2 v) {
    asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(a), "r"(v.x), "r"(v.y));
}
__device__ __forceinline__ void st_s128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w));
}

// mbarrier arrive by the lanes where `pred` holds (predicated, no branch).
__device__ __forceinline__ void mbar_arrive_if(uint64_t *bar, bool pred) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %1, 0;\n\t@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(
            smem_addr(bar)),
        "r"((uint32_t)pred)
        : "memory");
}


}  // namespace dqk
