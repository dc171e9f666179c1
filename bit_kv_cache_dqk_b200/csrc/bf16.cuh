// bf16.cuh -- the BF16 comparison decode: a paged BF16 K/V cache with no
// transform, no quantization and no channel pruning, the baseline Dual-QK's
// decode speedup is measured against ("Throughput on SGLang": the 3.75x over
// BF16 attention).  Same cooperative launch, work split, producer warp,
// records and log-sum-exp merge as k_decode, without its prologue; the
// consumers are plain bf16 tensor-core flash decoding.
//
// Block of (page, kv head): K [16][d] then V [16][d], BF16, row-major per
// token, with the 16-byte chunk x of row t stored at chunk position x ^ (t & 7)
// so that ldmatrix reads of 8 rows hit 8 different bank groups.
#pragma once

#include "attend.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "ptx.cuh"

namespace dqk {

constexpr int kB16Warps = 8;                   // consumer warps, one page of one kv head per stage each
constexpr int kB16StageBlocks = kB16Warps;     // (page, kv head) blocks per stage
constexpr int kB16Threads = 32 * (kB16Warps + 1);

__host__ __device__ constexpr int b16_block_bytes(int d) { return 2 * kPage * d * 2; }

// Byte offset of element (token t, channel c) of K (is_v = 0) or V in a block.
__host__ __device__ __forceinline__ int b16_offset(int d, int t, int c, int is_v) {
    const int x = c >> 3;
    return is_v * kPage * 2 * d + t * 2 * d + ((x ^ (t & 7)) << 4) + ((c & 7) << 1);
}

// ---------------------------------------------------------------------------
// append: copy rows into their blocks.  One CTA per (new row, kv head), one
// thread per 16-byte chunk of the K or V row.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(2 * D / 8) k_append_b16(const void *__restrict__ kin, const void *__restrict__ vin,
                                                         int dtype, const int *__restrict__ new_lens,
                                                         const int *__restrict__ seq_before,
                                                         const int *__restrict__ page_table, int max_pages,
                                                         int max_new, uint8_t *__restrict__ pool, long long num_pages,
                                                         int hkv) {
    constexpr int kChunks = D / 8;
    const int j = blockIdx.y;
    const int b = blockIdx.x / max_new, t = blockIdx.x - b * max_new;
    const int n = new_lens[b];
    if (t >= n) return;
    const int L0 = seq_before[b];
    const int pos = L0 + t, page = pos / kPage, slot = pos - page * kPage;
    const int phys = (L0 >= 0 && page < max_pages) ? page_table[(size_t)b * max_pages + page] : -1;
    if (phys < 0 || phys >= num_pages) {
        if (threadIdx.x == 0) dqk_flag_error(kErrBounds);
        return;
    }
    int row0 = 0;
    for (int bb = threadIdx.x & 31; bb < b; bb += 32) row0 += new_lens[bb];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) row0 += __shfl_xor_sync(0xffffffffu, row0, o);
    const int is_v = threadIdx.x / kChunks, x = threadIdx.x % kChunks;
    const size_t src = (((size_t)row0 + t) * hkv + j) * D + 8 * x;
    const void *in = is_v ? vin : kin;
    uint4 v;
    if (dtype == DQK_BF16) {
        v = *reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(in) + src);
    } else {
        const float4 a = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(in) + src);
        const float4 c = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(in) + src + 4);
        v = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
    }
    uint8_t *blk = pool + ((size_t)phys * hkv + j) * b16_block_bytes(D);
    *reinterpret_cast<uint4 *>(blk + b16_offset(D, slot, 8 * x, is_v)) = v;
}

// ---------------------------------------------------------------------------
// query fragments: qs = q * log2(e)/sqrt(d) as bf16 hi + lo pieces in the
// B operand of the m16n8k16 score tiles: per lane the registers of k-step s
// (channels 16s + 2*tig (+1), +8) for column n = gid: query head 4*nt + gid/2,
// piece gid & 1.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t b16_query_piece(const void *q, int dtype, size_t idx, float qscale, int pc) {
    const float x = ((dtype == DQK_BF16) ? bf16_to_f32(reinterpret_cast<const uint16_t *>(q)[idx])
                                         : reinterpret_cast<const float *>(q)[idx]) * qscale;
    const uint32_t hi = f32_to_bf16_rne(x);
    if (pc == 0) return hi;
    return f32_to_bf16_rne(x - __uint_as_float(hi << 16));
}

// ---------------------------------------------------------------------------
// attend
// ---------------------------------------------------------------------------
template <int D, int G>
struct B16State {
    static constexpr int NT = G > 4 ? 2 : 1;
    static constexpr int NM = D / 16;
    uint2 qf[NT][D / 16];          // score B fragments of this warp's (sequence, kv head)
    float m_run[NT];               // running max (log2 units) of this thread's head
    float oacc[NT][NM][4];         // PV accumulators: columns 2*tig (hi piece), 2*tig+1 (lo piece) of head tig
    float lacc[NT][4];             // row 0: softmax denominator (hi, lo pieces)
};

// One page (16 tokens, first nv valid) of the warp's kv head at shared address blk.
template <int D, int G, bool MASKED>
__device__ __forceinline__ void consume_b16(uint32_t blk, int nv, B16State<D, G> &st, int lane) {
    constexpr int NT = B16State<D, G>::NT, NM = B16State<D, G>::NM;
    const int gid = lane >> 2, tig = lane & 3;
    const int mi = lane >> 3, r8 = lane & 7;
    // scores: tokens x (head, piece) columns
    float c[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[nt][e] = 0.0f;
    {
        const int t = r8 + 8 * (mi & 1);
        const uint32_t rowk = blk + t * 2 * D;
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
            uint32_t a[4];
            ldmatrix_x4(a, rowk + (((2 * s + (mi >> 1)) ^ (t & 7)) << 4));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16(c[nt], a[0], a[1], a[2], a[3], st.qf[nt][s].x, st.qf[nt][s].y);
        }
    }
    float s0[NT], s1[NT];
    bool grow = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        s0[nt] = c[nt][0] + c[nt][1];   // token gid, head 4nt + tig
        s1[nt] = c[nt][2] + c[nt][3];   // token gid + 8
        if constexpr (MASKED) {
            if (gid >= nv) s0[nt] = -INFINITY;
            if (gid + 8 >= nv) s1[nt] = -INFINITY;
        }
        grow |= (s0[nt] > st.m_run[nt]) | (s1[nt] > st.m_run[nt]);
    }
    if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float mx = fmaxf(s0[nt], s1[nt]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mnew = fmaxf(st.m_run[nt], mx);
            const float alpha = fast_exp2(st.m_run[nt] - mnew);
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int e = 0; e < 4; ++e) st.oacc[nt][m][e] *= alpha;
#pragma unroll
            for (int e = 0; e < 4; ++e) st.lacc[nt][e] *= alpha;
            st.m_run[nt] = mnew;
        }
    }
    // P as bf16 hi + lo pieces in the PV B layout (column gid: head gid/2, piece gid&1)
    const int srcA = (2 * tig) * 4 + (gid >> 1);
    const bool lo_col = gid & 1;
    uint32_t pb0[NT], pb1[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const float p0 = fast_exp2(s0[nt] - st.m_run[nt]), p1 = fast_exp2(s1[nt] - st.m_run[nt]);
        const uint32_t hi = pack_bf16x2(p0, p1);
        const uint32_t lo = pack_bf16x2(p0 - __uint_as_float(hi << 16), p1 - __uint_as_float(hi & 0xffff0000u));
        const uint32_t w0h = __shfl_sync(0xffffffffu, hi, srcA), w1h = __shfl_sync(0xffffffffu, hi, srcA + 4);
        const uint32_t w0l = __shfl_sync(0xffffffffu, lo, srcA), w1l = __shfl_sync(0xffffffffu, lo, srcA + 4);
        const uint32_t w0 = lo_col ? w0l : w0h, w1 = lo_col ? w1l : w1h;
        pb0[nt] = prmt(w0, w1, 0x5410u);   // tokens 2tig, 2tig+1
        pb1[nt] = prmt(w0, w1, 0x7632u);   // tokens 2tig+8, 2tig+9
        // denominator: a row of ones
        const uint32_t ones = gid == 0 ? 0x3F803F80u : 0u;
        mma_bf16(st.lacc[nt], ones, 0u, ones, 0u, pb0[nt], pb1[nt]);
    }
    // values: O^T[c, col] += V^T[c, t] P[t, col]
    uint32_t vmask_lo = 0xffffffffu, vmask_hi = 0xffffffffu;
    if constexpr (MASKED) {
        // rows past the end of the sequence hold stale bytes: zero them
        vmask_lo = (2 * tig < nv ? 0x0000ffffu : 0u) | (2 * tig + 1 < nv ? 0xffff0000u : 0u);
        vmask_hi = (2 * tig + 8 < nv ? 0x0000ffffu : 0u) | (2 * tig + 9 < nv ? 0xffff0000u : 0u);
    }
    const int tv = r8 + 8 * (mi >> 1);
    const uint32_t rowv = blk + kPage * 2 * D + tv * 2 * D;
#pragma unroll
    for (int m = 0; m < NM; ++m) {
        uint32_t a[4];
        ldmatrix_x4_trans(a, rowv + (((2 * m + (mi & 1)) ^ (tv & 7)) << 4));
        if constexpr (MASKED) {
            a[0] &= vmask_lo;
            a[1] &= vmask_lo;
            a[2] &= vmask_hi;
            a[3] &= vmask_hi;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16(st.oacc[nt][m], a[0], a[1], a[2], a[3], pb0[nt], pb1[nt]);
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kB16Threads, 1) k_decode_b16(const __grid_constant__ DecodeParams dp) {
    const AttendParams &p = dp.a;
    using St = B16State<D, G>;
    constexpr int NT = St::NT, NM = St::NM;
    extern __shared__ __align__(128) unsigned char b16_smem[];
    const int S = p.stages;
    const uint32_t stage_bytes = (uint32_t)(kB16StageBlocks * p.bb);
    unsigned char *stage_mem = b16_smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(b16_smem + (size_t)S * stage_bytes);
    uint64_t *empty = full + kMaxStages;
    unsigned char *valid = reinterpret_cast<unsigned char *>(full) + kBarBytes;   // [kMaxStages][kB16StageBlocks]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(valid + kMaxStages * kB16StageBlocks);
    MergeHead *plan = reinterpret_cast<MergeHead *>(valid + kMaxStages * kB16StageBlocks + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = p.batch * p.nchunks;
    const int pps = p.pps;
    grid_dependency_wait();
    __shared__ CtaUnits sh_cu;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kB16Warps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        const CtaUnits c = cta_units(p.seq_lens, p.nchunks, R, blockIdx.x, p.num_ctas, lane);
        if (lane == 0) sh_cu = c;
    }
    __syncthreads();
    const CtaUnits cu = sh_cu;
    const int u0 = cu.u0, u1 = cu.u1;
    const int iters = (u1 - u0 + pps - 1) / pps;
    if (warp == kB16Warps) {
        const ProducerGate gate{nullptr, kMaxStages, nullptr, nullptr, 0, dp.ring_wait_ns};
        attend_producer<false>(p, stage_mem, full, empty, valid, abort_flag, S, stage_bytes, kB16StageBlocks, cu, iters,
                               lane, gate);
        return;
    }
    // consumer warp: kv head jl of the chunk, page slot pi of each stage
    const int jl = warp % p.hc, pi = warp / p.hc;
    const int gid = lane >> 2, tig = lane & 3;
    const int slot_base = (int)blockIdx.x;
    if (u1 > u0) init_records(p, cu, slot_base, pi, jl, G, D, lane);
    {
        const MergeHead mh = merge_head_of(p, cu.U, kB16Warps, warp, lane, 0);
        if (lane == 0) plan[warp] = mh;
    }

    int r = cu.r, ur = cu.ur;
    int npr = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
    int cur_run = -1, run_end = -1, partial_u = -1, nv_last = kPage;
    St st;
    auto start_run = [&](int rr) {
        const int b = rr / p.nchunks, chunk = rr - b * p.nchunks;
        const int j = chunk * p.hc + jl;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int hl = 4 * nt + (gid >> 1), pc = gid & 1;
            const size_t row = ((size_t)b * p.hq + (size_t)j * G + hl) * D;
#pragma unroll
            for (int s = 0; s < D / 16; ++s) {
                const int c0 = 16 * s + 2 * tig;
                uint2 f = make_uint2(0u, 0u);
                if (hl < G) {
                    f.x = b16_query_piece(dp.q, dp.q_dtype, row + c0, dp.qscale, pc) |
                          (b16_query_piece(dp.q, dp.q_dtype, row + c0 + 1, dp.qscale, pc) << 16);
                    f.y = b16_query_piece(dp.q, dp.q_dtype, row + c0 + 8, dp.qscale, pc) |
                          (b16_query_piece(dp.q, dp.q_dtype, row + c0 + 9, dp.qscale, pc) << 16);
                }
                st.qf[nt][s] = f;
            }
            st.m_run[nt] = -INFINITY;
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int e = 0; e < 4; ++e) st.oacc[nt][m][e] = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; ++e) st.lacc[nt][e] = 0.0f;
        }
        cur_run = rr;
    };
    auto finish_run = [&](int rr) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float l = __shfl_sync(0xffffffffu, st.lacc[nt][0] + st.lacc[nt][1], tig);
            const int hh = 4 * nt + tig;
            if (hh < G) {
                float *rec = p.part + record_index(slot_base + rr, pi, jl, hh, p.pw, p.hc, G) * rec_stride(D);
                if (gid == 0) {
                    rec[0] = st.m_run[nt];
                    rec[1] = l;
                }
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    rec[kRecHead + 16 * m + gid] = st.oacc[nt][m][0] + st.oacc[nt][m][1];
                    rec[kRecHead + 16 * m + gid + 8] = st.oacc[nt][m][2] + st.oacc[nt][m][3];
                }
            }
        }
    };
    auto switch_run = [&](int u) {
        if (cur_run >= 0) finish_run(cur_run);
        while (r < R && u >= ur + npr) {
            ur += npr;
            ++r;
            npr = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
        }
        start_run(r);
        run_end = ur + npr;
        const int Lb = p.seq_lens[r / p.nchunks];
        partial_u = (Lb & (kPage - 1)) ? run_end - 1 : -1;
        nv_last = Lb - (npr - 1) * kPage;
    };

    bool ok = true;
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t blk0 = smem_addr(stage_mem) + (uint32_t)((pi * p.hc + jl) * p.bb);
    for (int it = 0; it < iters; ++it) {
        if (!mbar_wait_bounded(&full[stage], phase, dp.ring_wait_ns)) {
            if (lane == 0) {
                *abort_flag = 1;
                dqk_flag_error(kErrTimeout);
            }
            ok = false;
            break;
        }
        const int ua = u0 + it * pps + pi;
        if (ua < u1 && valid[stage * kB16StageBlocks + pi]) {
            if (ua >= run_end) switch_run(ua);
            const uint32_t blk = blk0 + (uint32_t)stage * stage_bytes;
            if (ua == partial_u) consume_b16<D, G, true>(blk, nv_last, st, lane);
            else consume_b16<D, G, false>(blk, kPage, st, lane);
        }
        __syncwarp();
        mbar_arrive_if(&empty[stage], lane == 0);
        if (++stage == S) {
            stage = 0;
            phase ^= 1u;
        }
    }
    if (ok && cur_run >= 0) finish_run(cur_run);

    consumers_grid_sync<kB16Warps>(dp.grid_wait_ns, nullptr);
    grid_dependents_launch();
    merge_heads<D>(dp, cu.U, kB16Warps, warp, lane, reinterpret_cast<float *>(stage_mem), plan);
}

}  // namespace dqk
