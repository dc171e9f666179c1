// decode.cuh -- k_decode: one decode call of Dual-QK (and a decode step's
// cache append) as one cooperative kernel, one CTA per SM.
//
//   prologue   the consumer warps of every CTA take a share of the call's
//              small tasks -- the query transform and channel selection of
//              each query head ("Why the cache becomes a bottleneck":
//              query-channel pruning) and, in a decode step, the append of the
//              step's new K/V rows ("Paired transforms instead of shared
//              rotation": key transform, INT2 storage) -- while the producer
//              warp already streams the CTA's first pages (pages the append
//              writes wait for it);
//   grid barrier
//   attend     split-K pruned attention over the CTA's pages ("Throughput on
//              SGLang": 40 % of key channels dropped from reads, 2 bits per
//              stored value), one (m, l, o) record per (run, warp, head);
//   grid barrier
//   merge      the log-sum-exp merge of each query head's records, heads
//              spread over the CTAs (flash decoding's combine; the pages say
//              nothing about how the context is split).
//
// The grid barriers use the barrier word the driver provides to cooperative
// launches, so the kernel keeps no state of its own between calls and the
// workspace needs no initialisation.
#pragma once

#include "append.cuh"
#include "attend.cuh"
#include "common.cuh"
#include "ptx.cuh"
#include "qprep.cuh"

namespace dqk {

// Everything a decode launch needs besides the streaming parameters, passed
// as one __grid_constant__ kernel parameter.
struct DecodeParams {
    AttendParams a;
    uint8_t *pool_w;             // the pool, for the step's appends
    // query prep
    const float *t_q;
    const void *q;
    int q_dtype, pct;
    float qscale;
    int16_t *sel_out;
    // outputs: out [B][Hq][D], or (partial_out) records [B][Hq][2 + D]
    float *out;
    int partial_out;
    // the step's append (max_new > 0): new K/V rows, keys transformed by T_K
    const float *t_k;
    const void *k_in, *v_in;
    int kv_dtype, max_new;
    const int *new_lens, *seq_before;
    // bounds of the ring waits and of the grid barriers; test-only stall
    unsigned long long ring_wait_ns, grid_wait_ns;
    int stall;
    // shared memory between the ring and the barriers (bytes, a multiple of 16)
    int tail;
};

constexpr int kBarRing = 1, kBarConsumers = 2, kBarSlot0 = 3, kBarBusy = 4;   // named barriers (0 is __syncthreads)
constexpr int kFuseMaxNew = 4;   // decode steps append up to this many rows per sequence inside the kernel

// Shared memory besides the ring: full[kMaxStages], empty[kMaxStages], opened
// (and one spare word), valid flags [kMaxStages][stage blocks], abort flag (16 B), the merge
// plan (one MergeHead per consumer warp), then the per-warp score fragments
// of two-tile (G = 8) kernels.
constexpr int kBarBytes = (2 * kMaxStages + 2) * 8;
constexpr int kPlanBytes = 16 * 32 + 32;   // MergeHead per warp, then the CTA's CtaUnits
__host__ __device__ constexpr size_t decode_fixed_smem(int stage_blocks, int warps, int NT, int NG) {
    return (size_t)kBarBytes + (size_t)kMaxStages * stage_blocks + 16 + kPlanBytes +
           (NT > 1 ? (size_t)warps * NT * NG * (32 * 8 + 4 * 16) : 0);
}

// Shared memory of an append task (16-byte aligned): T_K[j] in padded rows,
// the key rows [D][kFuseMaxNew] fp64 (i-major), the store images of one row.
template <int D, int NS>
__host__ __device__ constexpr size_t append_scratch_bytes() {
    return (size_t)D * pad_row_bytes<D>() + (size_t)kFuseMaxNew * D * 8 + sizeof(RowStoreScratch<D, NS, 1>);
}

// Prologue scratch of one task (the largest of the two kinds) plus its
// 16-byte alignment.
template <int D, int NS>
__host__ __device__ constexpr size_t prologue_scratch_bytes(int G) {
    const size_t a = qprep_scratch_bytes<D>(G), b = append_scratch_bytes<D, NS>();
    return (a > b ? a : b) + 16;
}

// The rows sequence b appends in this launch (at most kFuseMaxNew), kv head
// j, by the NTH consumer threads of the CTA: T_K[j] staged like T_Q in the
// query task, then thread c < D computes k'_c of every row (interleaved fp64
// sequential sums) and the D threads quantize and store the rows one after
// the other -- the arithmetic, hence the bytes, of k_append_rows.
template <int D, int NS, int NTH, typename Meanwhile>
__device__ void append_kv(const DecodeParams &dp, int b, int j, int t, unsigned char *scratch, Meanwhile meanwhile) {
    const AttendParams &p = dp.a;
    constexpr int nthreads = NTH;
    const int n = min(dp.new_lens[b], kFuseMaxNew);
    if (n <= 0) return;   // uniform over the CTA
    const int L0 = dp.seq_before[b], lane = t & 31;
    double *xs = reinterpret_cast<double *>(scratch + (size_t)D * pad_row_bytes<D>());   // [D][kFuseMaxNew]
    RowStoreScratch<D, NS, 1> &S = *reinterpret_cast<RowStoreScratch<D, NS, 1> *>(xs + kFuseMaxNew * D);
    named_bar_sync(kBarConsumers, nthreads);   // the previous task is done with the scratch
    // T_K[j] and the key rows: every load in flight before the first store
    RowStage<D, NTH> rows;
    rows.load(dp.t_k + (size_t)j * D * D, t);
    int row0 = 0;   // rows of sequences 0..b-1 come first
    for (int bb = lane; bb < b; bb += 32) row0 += dp.new_lens[bb];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) row0 += __shfl_xor_sync(0xffffffffu, row0, o);
    constexpr int XN = (kFuseMaxNew * D + NTH - 1) / NTH;
    float xv[XN];
#pragma unroll
    for (int k = 0; k < XN; ++k) {
        const int i = t + k * NTH, r = i / D, c = i - r * D;
        xv[k] = (i < kFuseMaxNew * D && r < n)
                    ? load_elem_vol(dp.k_in, dp.kv_dtype, (((size_t)row0 + r) * p.hkv + j) * D + c)
                    : 0.0f;
    }
    rows.store(scratch, t);
#pragma unroll
    for (int k = 0; k < XN; ++k) {
        const int i = t + k * NTH, r = i / D, c = i - r * D;
        if (i < kFuseMaxNew * D) xs[c * kFuseMaxNew + r] = (double)xv[k];
    }
    named_bar_sync(kBarConsumers, nthreads);
    if (t >= D) {
        meanwhile();
        return;
    }
    const int c = t;
    double acc[kFuseMaxNew];
    dot_rows_pad<D, kFuseMaxNew>(scratch, c, xs, kFuseMaxNew, acc);
#pragma unroll
    for (int r = 0; r < kFuseMaxNew; ++r) {
        if (r >= n) break;   // uniform
        const float kp[1] = {__double2float_rn(acc[r])};
        const float xv[1] = {load_elem(dp.v_in, dp.kv_dtype, (((size_t)row0 + r) * p.hkv + j) * D + c)};
        const int page = (L0 + r) / kPage;
        const int phys[1] = {(L0 >= 0 && page < p.max_pages) ? p.page_table[(size_t)b * p.max_pages + page] : -1};
        quantize_store_rows<D, NS, 1>(kp, xv, phys, 1, L0 + r, c, dp.pool_w, p.num_pages, p.hkv, j, p.v_ch0, S,
                                      [] { named_bar_sync(kBarSlot0, D); });
    }
}

// CTA owning unit u of U split over C CTAs (32-bit arithmetic when it fits),
// and whether CTA c owns any unit.
__device__ __forceinline__ int cta_of_unit32(int u, int U, int C) {
    return U <= 0x7fffffff / (C + 1) ? ((u + 1) * C - 1) / U : (int)cta_of_unit(u, U, C);
}
__device__ __forceinline__ bool cta_has_units(int c, int U, int C) {
    return (long long)c * U / C < ((long long)c + 1) * U / C;
}

// Start unit of run r (sum of the pages of runs 0..r-1); warp-collective.
__device__ __forceinline__ int warp_run_start(const int *seq_lens, int nchunks, int r, int lane) {
    int base = 0;
    for (int r0 = 0; r0 < r; r0 += 32) {
        const int rr = r0 + lane;
        int np = rr < r ? run_pages(seq_lens, nchunks, rr) : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) np += __shfl_xor_sync(0xffffffffu, np, o);
        base += np;
    }
    return base;
}

// Log-sum-exp merge of the records of the query heads this CTA owns (head
// index b*Hq + h congruent to the CTA index modulo the grid):
//   out = sum_i o_i 2^(m_i - M) / sum_i l_i 2^(m_i - M), M = max_i m_i,
// over the records of every CTA (and page slot) that held pages of the
// head's run; with partial_out the merged (M, l, o) record instead.  The
// warps of a head take its records in turn, kMergeBatch at a time with all
// their loads in flight, then the first warp merges the warps' results in
// warp order: the result does not depend on timing.
//
// Record i (0 <= i < nrec) of a head is the one of CTA cf + i / pw, page slot
// i % pw, whose index (record_index) is linear in i: (i + (cf + r) pw) hc G +
// jl G + hh.  Which head a warp merges in the first round, and its record
// range, are worked out before the attend loop (MergeHead in shared memory).
constexpr int kMergeBatch = 8;

struct MergeHead {
    int hidx;     // b * Hq + h, -1: no head for this warp
    int np;       // pages of the head's run (0: empty sequence)
    int nrec;     // records of the run
    int rbase;    // (cf + r) * pw
    int off;      // jl * G + hh
    int dense;    // every CTA owns units (all records exist)
    int cf;       // first CTA holding pages of the run
    int pad;
};

// The head warp `warp` merges in round k0 (warp-collective).
__device__ __forceinline__ MergeHead merge_head_of(const AttendParams &p, int U, int W, int warp, int lane, int k0) {
    MergeHead mh{-1, 0, 0, 0, 0, 1, 0, 0};
    const int C = gridDim.x, H = p.batch * p.hq, G = p.hq / p.hkv;
    const int mine = (int)blockIdx.x < H ? (H - 1 - (int)blockIdx.x) / C + 1 : 0;
    if (mine == 0) return mh;
    const int nconc = min(mine, W), wpr = W / nconc, gi = warp / wpr;
    const int k = k0 + gi;
    if (gi >= nconc || k >= mine) return mh;
    mh.hidx = (int)blockIdx.x + C * k;
    const int b = mh.hidx / p.hq, h = mh.hidx - b * p.hq;
    const int j = h / G, chunk = j / p.hc, jl = j - chunk * p.hc, hh = h - j * G;
    const int r = b * p.nchunks + chunk;
    mh.np = run_pages(p.seq_lens, p.nchunks, r);
    mh.off = jl * G + hh;
    mh.dense = U >= C ? 1 : 0;
    if (mh.np > 0) {
        const int ur = warp_run_start(p.seq_lens, p.nchunks, r, lane);
        const int cf = cta_of_unit32(ur, U, C), cl = cta_of_unit32(ur + mh.np - 1, U, C);
        mh.nrec = (cl - cf + 1) * p.pw;
        mh.rbase = (cf + r) * p.pw;
        mh.cf = cf;
    }
    return mh;
}

template <int D>
__device__ void merge_heads(const DecodeParams &dp, int U, int W, int warp, int lane, float *sm,
                            const MergeHead *plan) {
    const AttendParams &p = dp.a;
    constexpr int V = D / 32;   // channels per lane
    const int C = gridDim.x, H = p.batch * p.hq, G = p.hq / p.hkv;
    const int mine = (int)blockIdx.x < H ? (H - 1 - (int)blockIdx.x) / C + 1 : 0;
    if (mine == 0) return;
    const int nconc = min(mine, W);          // heads merged at once
    const int wpr = W / nconc;               // warps per head
    const int wl = warp % wpr;
    const size_t istride = (size_t)p.hc * G;
#pragma unroll 1
    for (int k0 = 0; k0 < mine; k0 += nconc) {
        const MergeHead mh = k0 == 0 ? plan[warp] : merge_head_of(p, U, W, warp, lane, k0);
        float M = -INFINITY, Ls = 0.0f, O[V];
#pragma unroll
        for (int e = 0; e < V; ++e) O[e] = 0.0f;
        if (mh.hidx >= 0) {
#pragma unroll 1
            for (int i0 = wl; i0 < mh.nrec; i0 += kMergeBatch * wpr) {
                float m[kMergeBatch], l[kMergeBatch], o[kMergeBatch][V];
#pragma unroll
                for (int q = 0; q < kMergeBatch; ++q) {
                    const int i = i0 + q * wpr;
                    m[q] = -INFINITY;
                    l[q] = 0.0f;
#pragma unroll
                    for (int e = 0; e < V; ++e) o[q][e] = 0.0f;
                    if (i < mh.nrec && (mh.dense || cta_has_units(mh.cf + i / p.pw, U, C))) {
                        const float *rec =
                            p.part + ((size_t)(i + mh.rbase) * istride + mh.off) * rec_stride(D);
                        m[q] = __ldcg(rec);
                        l[q] = __ldcg(rec + 1);
                        if constexpr (V == 4) {
                            const float4 v4 = __ldcg(reinterpret_cast<const float4 *>(rec + kRecHead) + lane);
                            o[q][0] = v4.x; o[q][1] = v4.y; o[q][2] = v4.z; o[q][3] = v4.w;
                        } else {
                            const float2 v2 = __ldcg(reinterpret_cast<const float2 *>(rec + kRecHead) + lane);
                            o[q][0] = v2.x; o[q][1] = v2.y;
                        }
                    }
                }
                float Mn = M;
#pragma unroll
                for (int q = 0; q < kMergeBatch; ++q) Mn = fmaxf(Mn, m[q]);
                if (Mn == -INFINITY) continue;
                const float sc = exp2f(M - Mn);   // 0 while M is -inf
                Ls *= sc;
#pragma unroll
                for (int e = 0; e < V; ++e) O[e] *= sc;
                M = Mn;
#pragma unroll
                for (int q = 0; q < kMergeBatch; ++q) {
                    const float w = m[q] == -INFINITY ? 0.0f : exp2f(m[q] - M);   // empty record: no o values
                    Ls = fmaf(w, l[q], Ls);
#pragma unroll
                    for (int e = 0; e < V; ++e) O[e] = w != 0.0f ? fmaf(w, o[q][e], O[e]) : O[e];
                }
            }
            float *row = sm + (size_t)warp * (D + 4);
            if (lane == 0) {
                row[0] = M;
                row[1] = Ls;
            }
#pragma unroll
            for (int e = 0; e < V; ++e) row[4 + V * lane + e] = O[e];
        }
        named_bar_sync(kBarConsumers, 32 * W);
        if (mh.hidx >= 0 && wl == 0) {
            float Mt = -INFINITY, Lt = 0.0f, Ot[V];
#pragma unroll
            for (int e = 0; e < V; ++e) Ot[e] = 0.0f;
#pragma unroll 1
            for (int w = warp; w < warp + wpr; ++w) {
                const float *row = sm + (size_t)w * (D + 4);
                const float m = row[0];
                if (m == -INFINITY) continue;
                const float Mn = fmaxf(Mt, m);
                const float sc = exp2f(Mt - Mn), wgt = exp2f(m - Mn);
                Lt = fmaf(wgt, row[1], Lt * sc);
#pragma unroll
                for (int e = 0; e < V; ++e) Ot[e] = fmaf(wgt, row[4 + V * lane + e], Ot[e] * sc);
                Mt = Mn;
            }
            const bool any = mh.np > 0;
            if (dp.partial_out) {
                float *pr = dp.out + (size_t)mh.hidx * (D + 2);
                if (lane == 0) {
                    pr[0] = any ? Mt : -INFINITY;
                    pr[1] = any ? Lt : 0.0f;
                }
#pragma unroll
                for (int e = 0; e < V; ++e) pr[2 + V * lane + e] = any ? Ot[e] : 0.0f;
            } else {
                const float inv = (any && Lt > 0.0f) ? 1.0f / Lt : 0.0f;
                float *o = dp.out + (size_t)mh.hidx * D + V * lane;
                if constexpr (V == 4) {
                    *reinterpret_cast<float4 *>(o) = make_float4(Ot[0] * inv, Ot[1] * inv, Ot[2] * inv, Ot[3] * inv);
                } else {
                    *reinterpret_cast<float2 *>(o) = make_float2(Ot[0] * inv, Ot[1] * inv);
                }
            }
        }
        named_bar_sync(kBarConsumers, 32 * W);
    }
}

// The CTA's bookkeeping before the attend loop: the unit range (written to
// shared memory), the empty records of each consumer warp's runs and each
// warp's merge plan.  A functor holding plain values, so that nothing of the
// caller's is address-taken.  Run by every consumer warp for itself (all of
// them idle), or, inside a prologue task, by the warps the task leaves idle
// (warps >= first) for every consumer warp in turn.
template <int D, int G>
struct Bookkeeping {
    const AttendParams *p;
    CtaUnits *cu_sm;
    MergeHead *plan;
    int R, warp, lane, first;
    __device__ __forceinline__ void for_warp(const CtaUnits &cu, int w) const {
        const int jl = w % p->hc, pi = w / p->hc;
        if (cu.u1 > cu.u0) init_records(*p, cu, (int)blockIdx.x, pi, jl, G, D, lane);
        const MergeHead mh = merge_head_of(*p, cu.U, attend_warps(G), w, lane, 0);
        if (lane == 0) plan[w] = mh;
    }
    __device__ __forceinline__ void operator()() const {
        if (warp < first) return;
        const CtaUnits cu = cta_units(p->seq_lens, p->nchunks, R, blockIdx.x, p->num_ctas, lane);
        if (warp == first && lane == 0) *cu_sm = cu;
        for (int w = warp - first; w < attend_warps(G); w += attend_warps(G) - first) for_warp(cu, w);
    }
};
template <int D, int G>
struct BookkeepingOnce {
    const Bookkeeping<D, G> *bk;
    bool run;
    __device__ __forceinline__ void operator()() const {
        if (run) (*bk)();
    }
};

// The grid barrier between the phases, by the consumer warps of every CTA
// (the producer takes no part).  A barrier that times out (or a launch that
// was not cooperative) reports DQK_ERR_TIMEOUT; every CTA still arrives at
// every barrier, which keeps the driver's word consistent for later launches.
template <int W>
__device__ __forceinline__ void consumers_grid_sync(uint64_t limit_ns, uint64_t *opened) {
    named_bar_sync(kBarConsumers, 32 * W);
    if (threadIdx.x == 0) {
        unsigned int *word = coop_barrier_word();
        if (!(word && grid_sync_bounded(word, limit_ns))) dqk_flag_error(kErrTimeout);
        if (opened) mbar_arrive(opened);
    }
    named_bar_sync(kBarConsumers, 32 * W);
}

template <int D, int G, bool VCH0, int NS>
__global__ void __launch_bounds__(attend_threads(G), 1) k_decode(const __grid_constant__ DecodeParams dp) {
    const AttendParams &p = dp.a;
    using T = AttendTile<D, G>;
    constexpr int kConsumerWarps = attend_warps(G), kStageBlocks = attend_stage_blocks(G);
    constexpr int BPW = attend_pages_per_warp(G);
    static_assert(BPW >= 2 && BPW <= 8, "pages per warp");
    constexpr int NG = T::NG, NT = T::NT, NM = T::NM;
    extern __shared__ __align__(128) unsigned char attend_smem[];
    const int S = p.stages;
    const uint32_t stage_bytes = (uint32_t)(kStageBlocks * p.bb);
    unsigned char *stage_mem = attend_smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(attend_smem + (size_t)S * stage_bytes + dp.tail);
    uint64_t *empty = full + kMaxStages;
    uint64_t *opened = empty + kMaxStages;
    unsigned char *valid = reinterpret_cast<unsigned char *>(full) + kBarBytes;   // [kMaxStages][kStageBlocks]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(valid + kMaxStages * kStageBlocks);
    MergeHead *plan = reinterpret_cast<MergeHead *>(valid + kMaxStages * kStageBlocks + 16);
    // per consumer warp: QK B fragments [NT][NG][32] uint2, head constants [NT][NG][4] float4
    unsigned char *frag_mem = valid + kMaxStages * kStageBlocks + 16 + kPlanBytes;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = p.batch * p.nchunks;
    const int pps = p.pps;
    // launched with programmatic serialization: everything read below may come
    // from the kernel before this one on the stream
    grid_dependency_wait();

    // The producer initialises the ring's barriers and announces them on named
    // barrier kBarRing without waiting; producer and consumers work out the
    // CTA's unit range on their own, so the first copies wait on nothing but
    // the lengths and the page table, and the consumers' prologue on nothing.
    if (warp == kConsumerWarps) {
        if (lane == 0) {
            for (int s = 0; s < S; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], kConsumerWarps);
            }
            mbar_init(opened, 1);
            *abort_flag = 0;
            fence_mbar_init();
        }
        __syncwarp();
        named_bar_arrive(kBarRing, attend_threads(G));
    }
    // the prologue works in the last ring stages and the tail after them; the
    // producer fills those stages only once `opened` completes
    const uint32_t scratch_bytes = (uint32_t)prologue_scratch_bytes<D, NS>(G);
    const uint32_t tail = (uint32_t)dp.tail;
    const int scratch_stages =
        scratch_bytes > tail ? (int)((scratch_bytes - tail + stage_bytes - 1) / stage_bytes) : 0;
    unsigned char *scratch_raw = stage_mem + (size_t)(S - scratch_stages) * stage_bytes;
    unsigned char *scratch = scratch_raw + ((16u - (smem_addr(scratch_raw) & 15u)) & 15u);

    if (warp == kConsumerWarps) {
        const CtaUnits cu = cta_units(p.seq_lens, p.nchunks, R, blockIdx.x, p.num_ctas, lane);
        const int iters = (cu.u1 - cu.u0 + pps - 1) / pps;
        const ProducerGate gate{opened, S - scratch_stages, dp.max_new > 0 ? dp.new_lens : nullptr, dp.seq_before,
                                dp.stall, dp.ring_wait_ns};
        attend_producer<true>(p, stage_mem, full, empty, valid, abort_flag, S, stage_bytes, kStageBlocks, cu, iters,
                              lane, gate);
        return;
    }

    // ------------------------------------------------------------- prologue
    // tasks = [the step's appends (sequence, kv head)] + [query prep (sequence,
    // kv head)], task k on CTA k mod C, each by all consumer warps of the CTA;
    // the CTA's bookkeeping (unit range, empty records, merge plan; results in
    // shared memory) runs while the first task's loads are in flight
    CtaUnits *cu_sm = reinterpret_cast<CtaUnits *>(plan + 16);
    {
        // in a query task the first max(G, D/32) warps are busy and the others
        // do the bookkeeping of all warps meanwhile; in an append task the
        // warps past D/32 do (when there are none, each warp does its own
        // after the tasks)
        constexpr int kFirst = (D / 32 > G ? D / 32 : G);
        constexpr int kThreads = 32 * kConsumerWarps;
        const QueryOut qo{const_cast<uint2 *>(p.qf), const_cast<float *>(p.qk), const_cast<uint32_t *>(p.qm),
                          const_cast<float *>(p.q0), dp.sel_out};
        const int n_app = dp.max_new > 0 ? p.batch * p.hkv : 0;
        const int n_tasks = n_app + p.batch * p.hkv;
        bool done = false;
        for (int k = (int)blockIdx.x; k < n_tasks; k += (int)gridDim.x) {
            const Bookkeeping<D, G> bkk{&p, cu_sm, plan, R, warp, lane, k < n_app ? D / 32 : kFirst};
            const BookkeepingOnce<D, G> once{&bkk, !done && bkk.first < kConsumerWarps};
            if (k < n_app) {
                append_kv<D, NS, kThreads>(dp, k / p.hkv, k % p.hkv, threadIdx.x, scratch, once);
            } else {
                const int u = k - n_app;
                qprep_kv<D, G, kThreads>(dp.t_q, dp.q, dp.q_dtype, p.hq, p.hkv, dp.pct, dp.qscale, u / p.hkv,
                                         u % p.hkv, threadIdx.x, kBarConsumers, kBarBusy, scratch, qo, once);
            }
            done = done || bkk.first < kConsumerWarps;
        }
        if (!done) {   // no task, or none with idle warps: every warp for itself
            const Bookkeeping<D, G> own{&p, cu_sm, plan, R, warp, lane, 0};
            const CtaUnits cu = cta_units(p.seq_lens, p.nchunks, R, blockIdx.x, p.num_ctas, lane);
            if (warp == 0 && lane == 0) *cu_sm = cu;
            own.for_warp(cu, warp);
        }
        if (n_app) fence_proxy_async_global();   // appended rows are read by bulk copies
    }
    named_bar_sync(kBarRing, attend_threads(G));
    consumers_grid_sync<kConsumerWarps>(dp.grid_wait_ns, opened);
    const CtaUnits cu = *cu_sm;
    const int u0 = cu.u0, u1 = cu.u1;
    const int nunits = u1 - u0;
    const int iters = (nunits + pps - 1) / pps;
    const int jl = warp % p.hc, pi = warp / p.hc;   // kv head of the chunk, page group of each stage
    const int slot_base = (int)blockIdx.x;
    const int gid = lane >> 2, tig = lane & 3;

    // --------------------------------------------------------------- attend
    int r = cu.r, ur = cu.ur;
    int npr = r < R ? run_pages(p.seq_lens, p.nchunks, r) : 0;
    int cur_run = -1, run_end = -1, partial_u = -1, nv_last = kPage;
    int fast_end = -1;   // a stage's pages below this unit are full pages of the current run and the CTA

    WarpState<D, G> st;
    LaneOffsets lo;
    lo.lane16 = lane * 16;
    lo.gid8 = gid * 8;
    lo.kmin = gid * 2 * NG + (tig & (NG / 2 - 1)) * 4;   // in range for every lane (B rows past 2 NG are 0)
    lo.gid4 = gid * 4;
    lo.tig16 = tig * 16;
    lo.vmin = (tig * NS + (gid < NS ? gid : 0)) * 4;
    lo.srcA = (2 * tig) * 4 + (gid >> 1);
    {
        unsigned char *mine = frag_mem + (size_t)warp * NT * NG * (32 * 8 + 4 * 16);
        lo.sq = smem_addr(mine) + lane * 8;
        lo.sk = smem_addr(mine + NT * NG * 32 * 8) + tig * 16;
    }
    lo.ones_lane = gid == NS ? 0x3C003C00u : 0u;
    lo.vmin_mask = gid < NS ? 0xffffffffu : 0u;

    // query fragments were written by other CTAs in the prologue: read at L2
    auto start_run = [&](int rr) {
        const int b = rr / p.nchunks, chunk = rr - b * p.nchunks;
        const int j = chunk * p.hc + jl;
        const size_t bj = (size_t)b * p.hkv + j;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const uint2 qb = __ldcg(&p.qf[((bj * NT + nt) * NG + g) * 32 + lane]);
                const float kq = __ldcg(&p.qk[((bj * NT + nt) * (NG + 1) + g) * 4 + tig]) * (1.0f / 256.0f);
                if constexpr (WarpState<D, G>::kRegFrags) {
                    st.qb[g] = qb;
                    st.kq[g] = kq;
                } else {
                    st_s64(lo.sq + (nt * NG + g) * 256, qb);
                    if (gid == 0) st_s32(lo.sk + (nt * NG + g) * 64, __float_as_uint(kq));
                }
            }
            st.sgh[nt] = __ldcg(&p.qk[((bj * NT + nt) * (NG + 1) + NG) * 4 + tig]);
            __syncwarp();
            st.qmin[nt] = __ldcg(&p.qm[(bj * NT + nt) * 32 + lane]);
            const int hh = 4 * nt + tig;
            st.q0v[nt] = hh < G ? __ldcg(&p.q0[(size_t)b * p.hq + j * G + hh]) : 0.0f;
            st.m_run[nt] = -INFINITY;
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int e = 0; e < 4; ++e) st.oacc[nt][m][e] = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; ++e) st.macc[nt][e] = 0.0f;
        }
        cur_run = rr;
    };

    auto finish_run = [&](int rr) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float minterm[NS];
#pragma unroll
            for (int g = 0; g < NS; ++g) minterm[g] = __shfl_sync(0xffffffffu, st.macc[nt][0], g * 4 + tig);
            const float l = __shfl_sync(0xffffffffu, st.macc[nt][0], NS * 4 + tig);
            const float v0t = __shfl_sync(0xffffffffu, st.macc[nt][0], (NS + 1) * 4 + tig);
            const int hh = 4 * nt + tig;
            if (hh < G) {
                float *rec = p.part + record_index(slot_base + rr, pi, jl, hh, p.pw, p.hc, G) * rec_stride(D);
                if (gid == 0) {
                    rec[0] = st.m_run[nt];
                    rec[1] = l;
                }
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    const int c0 = 16 * m + gid, c1 = c0 + 8;
                    const float mt = minterm[NS == 1 ? 0 : (m >> 1)];
                    const float f = vfield_scale<NG>(m);
                    rec[kRecHead + c0] = (VCH0 && c0 == 0) ? v0t : fmaf(st.oacc[nt][m][0], f, mt);
                    rec[kRecHead + c1] = fmaf(st.oacc[nt][m][2], f, mt);
                }
            }
        }
    };

    // move to the run holding unit u (u >= run_end)
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
        fast_end = min(partial_u >= 0 ? partial_u : run_end, u1);
    };

    if (iters > 0) {
        switch_run(u0 + BPW * pi < u1 ? u0 + BPW * pi : u0);

        bool ok = true;
        int stage = 0;
        uint32_t phase = 0;
        const uint32_t blk_a = smem_addr(stage_mem) + (uint32_t)((BPW * pi * p.hc + jl) * p.bb);
        const uint32_t page_gap = (uint32_t)(p.hc * p.bb);
        // n (1 .. BPW-1) full pages of one run at shared addresses base + q * page_gap
        auto consume_batch = [&](int n, uint32_t base) {
            if constexpr (BPW >= 4) {
                if (n == 3) {
                    const uint32_t sb3[3] = {base, base + page_gap, base + 2 * page_gap};
                    consume<D, G, VCH0, NS, 3, false>(sb3, kPage, st, lane, lo);
                    return;
                }
            }
            if constexpr (BPW >= 3) {
                if (n == 2) {
                    const uint32_t sb2[2] = {base, base + page_gap};
                    consume<D, G, VCH0, NS, 2, false>(sb2, kPage, st, lane, lo);
                    return;
                }
            }
            const uint32_t sb1[1] = {base};
            consume<D, G, VCH0, NS, 1, false>(sb1, kPage, st, lane, lo);
        };

        const uint32_t valid_addr = smem_addr(valid) + BPW * pi;
        constexpr uint32_t kAllValid = (1u << BPW) - 1u;
        for (int it = 0; it < iters; ++it) {
            if (!mbar_wait_bounded(&full[stage], phase, dp.ring_wait_ns)) {
                if (lane == 0) {
                    *abort_flag = 1;
                    dqk_flag_error(kErrTimeout);
                }
                ok = false;
                break;
            }
            const int ua = u0 + it * pps + BPW * pi;
            if (ua < u1) {
                const uint32_t sa = blk_a + (uint32_t)stage * stage_bytes;
                const int ul = ua + BPW - 1;
                // flags of the warp's page slots (one byte each), as a bit mask
                const uint32_t va = valid_addr + stage * kStageBlocks;
                uint32_t vv = 0, vw = 0;
                if constexpr (BPW == 4) {
                    vw = ld_s32(va);
                    vv = (vw & 1u) | ((vw >> 7) & 2u) | ((vw >> 14) & 4u) | ((vw >> 21) & 8u);
                } else if constexpr (BPW == 2) {
                    vw = ld_s16(va);
                    vv = (vw & 1u) | ((vw >> 7) & 2u);
                } else {
#pragma unroll
                    for (int q = 0; q < BPW; ++q) vv |= ld_s8(va + q) << q;
                    vw = vv == kAllValid ? 0x01010101u : 0u;
                }
                constexpr uint32_t kAllValidBytes = BPW == 4 ? 0x01010101u : BPW == 2 ? 0x0101u : 0x01010101u;
                if (ua >= run_end) switch_run(ua);
                if (ul < fast_end && vw == kAllValidBytes) {
                    uint32_t sbb[BPW];
#pragma unroll
                    for (int q = 0; q < BPW; ++q) sbb[q] = sa + q * page_gap;
                    consume<D, G, VCH0, NS, BPW, false>(sbb, kPage, st, lane, lo);
                } else if (vv == kAllValid && ul < u1 && run_end <= ul && partial_u < 0) {
                    // the pages cross one run boundary, the run's last page is full:
                    // the pages of each run as one batch
                    const int k = run_end - ua;   // 1 .. BPW-1 pages of the current run
                    consume_batch(k, sa);
                    switch_run(run_end);
                    if (ul < run_end && !(partial_u >= ua + k && partial_u <= ul)) {
                        consume_batch(BPW - k, sa + (uint32_t)k * page_gap);
                    } else {
#pragma unroll
                        for (int q = 1; q < BPW; ++q) {
                            if (q < k) continue;
                            const int uq = ua + q;
                            if (uq >= run_end) switch_run(uq);
                            const uint32_t s1[1] = {sa + q * page_gap};
                            if (uq == partial_u) consume<D, G, VCH0, NS, 1, true>(s1, nv_last, st, lane, lo);
                            else consume<D, G, VCH0, NS, 1, false>(s1, kPage, st, lane, lo);
                        }
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < BPW; ++q) {
                        const int uq = ua + q;
                        if (uq >= u1) break;
                        if (uq >= run_end) switch_run(uq);
                        if ((vv >> q) & 1u) {
                            const uint32_t s1[1] = {sa + q * page_gap};
                            if (uq == partial_u) consume<D, G, VCH0, NS, 1, true>(s1, nv_last, st, lane, lo);
                            else consume<D, G, VCH0, NS, 1, false>(s1, kPage, st, lane, lo);
                        }
                    }
                }
            }
            __syncwarp();
            mbar_arrive_if(&empty[stage], lane == 0);
            if (++stage == S) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (ok && cur_run >= 0) finish_run(cur_run);
    }

    // ---------------------------------------------------------------- merge
    consumers_grid_sync<kConsumerWarps>(dp.grid_wait_ns, nullptr);
    grid_dependents_launch();
    merge_heads<D>(dp, cu_sm->U, kConsumerWarps, warp, lane, reinterpret_cast<float *>(stage_mem), plan);
}

}  // namespace dqk
