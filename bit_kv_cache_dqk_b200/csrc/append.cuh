// append.cuh -- k_quant_pack: key transform, INT2 quantization and packing of
// new K/V rows into the paged cache (the cache-write side of Dual-QK: "Paired
// transforms instead of shared rotation" -- partial key whitening, channel-0
// protection; "Throughput on SGLang" -- 2 bits per stored value).
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace dqk {

template <int D>
struct AppendSmem {
    static constexpr int NG = D / kGroup;
    static constexpr int kMaxBlockBytes = 8 * D + 128 * NG + 64;
    double tk[D * (D + 1)];          // T_K[j] in fp64, rows padded by one element
    double x[kPage][D];              // input K rows of the page's new slots, fp64
    float kp[kPage][D];              // their transformed rows k' (fp32)
    uint8_t kcode[kPage][D];         // plain codes of the page being rewritten
    uint8_t vcode[kPage][D];
    uint16_t kscale[kPage][NG], kmin[kPage][NG], kch0[kPage];
    uint16_t vscale[kPage][NG], vmin[kPage][NG], vch0[kPage];
    uint4 blk[kMaxBlockBytes / 16];  // the packed block
};

// One 32-channel group held by a warp (lane = channel of the group): group
// min/max of the fp32 values by warp shuffles (with -0 read as +0), then fp64
// arithmetic with single RNE roundings: scale = fp16((max - min) / 3), min =
// fp16(min), code = clamp(rne((x - min) / scale), 0, 3) (0 when scale is 0).
// excluded: this lane's value (channel 0 of a protected key) takes no part
// and gets code 0.
__device__ __forceinline__ void warp_minmax(float x, bool excluded, float &lo, float &hi) {
    lo = excluded ? __int_as_float(0x7f800000) : x;
    hi = excluded ? __int_as_float(0xff800000) : x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
}

// scale/min of a group from its range, and the code of x
__device__ __forceinline__ int quant_code(float x, bool excluded, float lo, float hi, uint16_t &sh, uint16_t &mh) {
    sh = f64_to_f16_rne(((double)hi - (double)lo) / 3.0);
    mh = f64_to_f16_rne((double)lo);
    const double s = f16_to_f64(sh), mn = f16_to_f64(mh);
    int code = 0;
    if (!excluded && s != 0.0) {
        const double r = rint(((double)x - mn) / s);
        code = r < 0.0 ? 0 : (r > 3.0 ? 3 : (int)r);
    }
    return code;
}

__device__ __forceinline__ int quantize_group(float xv, bool excluded, uint16_t &sh, uint16_t &mh) {
    const float x = xv + 0.0f;
    float lo, hi;
    warp_minmax(x, excluded, lo, hi);
    return quant_code(x, excluded, lo, hi, sh, mh);
}

// Quantize the D values a warp holds (lane owns channels lane + 32*m, i.e.
// channel `lane` of block m) into codes / fp16 scale / fp16 min / BF16 ch0,
// with NS scale groups (NG of 32 channels, or 1 over the whole row).
// protect: channel 0 goes to BF16, is excluded from group 0's range and its
// code is 0.
template <int NG, int NS>
__device__ __forceinline__ void quantize_warp(const float (&vals)[NG], bool protect, int lane,
                                              uint8_t *codes, uint16_t *scale, uint16_t *minv,
                                              uint16_t *ch0) {
    if constexpr (NS == 1) {
        float lo = __int_as_float(0x7f800000), hi = __int_as_float(0xff800000);
#pragma unroll
        for (int m = 0; m < NG; ++m) {
            float l, h;
            warp_minmax(vals[m] + 0.0f, protect && m == 0 && lane == 0, l, h);
            lo = fminf(lo, l);
            hi = fmaxf(hi, h);
        }
#pragma unroll
        for (int m = 0; m < NG; ++m) {
            uint16_t sh, mh;
            const int code = quant_code(vals[m] + 0.0f, protect && m == 0 && lane == 0, lo, hi, sh, mh);
            codes[m * kGroup + lane] = (uint8_t)code;
            if (lane == 0 && m == 0) {
                scale[0] = sh;
                minv[0] = mh;
            }
        }
    } else {
#pragma unroll
        for (int m = 0; m < NG; ++m) {
            uint16_t sh, mh;
            const int code = quantize_group(vals[m], protect && m == 0 && lane == 0, sh, mh);
            codes[m * kGroup + lane] = (uint8_t)code;
            if (lane == 0) {
                scale[m] = sh;
                minv[m] = mh;
            }
        }
    }
    if (lane == 0) *ch0 = protect ? f32_to_bf16_rne(vals[0]) : (uint16_t)0;
}

__device__ __forceinline__ float load_elem(const void *p, int dtype, size_t idx) {
    if (dtype == DQK_BF16) return bf16_to_f32(reinterpret_cast<const uint16_t *>(p)[idx]);
    return reinterpret_cast<const float *>(p)[idx];
}

// Block <-> plain arrays.  One thread per 32-bit code word.
template <int D>
__device__ void unpack_block(AppendSmem<D> &S, const Layout &L, int v_ch0) {
    constexpr int NG = D / kGroup;
    const uint32_t *w = reinterpret_cast<const uint32_t *>(S.blk);
    for (int widx = threadIdx.x; widx < 32 * NG; widx += blockDim.x) {
        const int lane = widx / NG, W = widx % NG, gid = lane >> 2, tig = lane & 3;
        const uint32_t word = w[(L.kc >> 2) + widx];
        // byte j, field f: group g = f % NG, register r = W + NG * (f / NG)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int f = 0; f < 4; ++f) {
                const int g = f % NG, r = W + NG * (f / NG);
                S.kcode[gid + 8 * (r & 1)][32 * g + 16 * (r >> 1) + 4 * tig + j] =
                    (uint8_t)((word >> (8 * j + 2 * f)) & 3u);
            }
    }
    const uint8_t *vb = reinterpret_cast<const uint8_t *>(S.blk) + L.vc;
    for (int idx = threadIdx.x; idx < kPage * D; idx += blockDim.x) {
        const int t = idx / D, c = idx % D;
        int off, bit;
        vcode_pos(NG, t, c, off, bit);
        S.vcode[t][c] = (uint8_t)((*reinterpret_cast<const uint32_t *>(vb + off) >> bit) & 3u);
    }
    const uint16_t *h = reinterpret_cast<const uint16_t *>(S.blk);
    const int ns = L.ns;
    for (int idx = threadIdx.x; idx < kPage * ns; idx += blockDim.x) {
        const int t = idx / ns, g = idx % ns;
        S.kscale[t][g] = h[(L.ks >> 1) + kscale_idx(ns, t, g)];
        S.kmin[t][g] = h[(L.km >> 1) + kscale_idx(ns, t, g)];
        S.vscale[t][g] = h[(L.vs >> 1) + vscale_idx(ns, t, g)];
        S.vmin[t][g] = h[(L.vm >> 1) + vscale_idx(ns, t, g)];
    }
    for (int t = threadIdx.x; t < kPage; t += blockDim.x) {
        S.kch0[t] = h[(L.k0 >> 1) + k0_idx(t)];
        S.vch0[t] = v_ch0 ? h[(L.v0 >> 1) + t] : (uint16_t)0;
    }
}

template <int D>
__device__ void pack_block(AppendSmem<D> &S, const Layout &L, int v_ch0) {
    constexpr int NG = D / kGroup;
    uint32_t *w = reinterpret_cast<uint32_t *>(S.blk);
    for (int widx = threadIdx.x; widx < 32 * NG; widx += blockDim.x) {
        const int lane = widx / NG, W = widx % NG, gid = lane >> 2, tig = lane & 3;
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int f = 0; f < 4; ++f) {
                const int g = f % NG, r = W + NG * (f / NG);
                word |= ((uint32_t)S.kcode[gid + 8 * (r & 1)][32 * g + 16 * (r >> 1) + 4 * tig + j] & 3u)
                        << (8 * j + 2 * f);
            }
        w[(L.kc >> 2) + widx] = word;
        w[(L.vc >> 2) + widx] = 0u;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < kPage * D; idx += blockDim.x) {
        const int t = idx / D, c = idx % D;
        int off, bit;
        vcode_pos(NG, t, c, off, bit);
        atomicOr(&w[(L.vc + off) >> 2], ((uint32_t)S.vcode[t][c] & 3u) << bit);
    }
    uint16_t *h = reinterpret_cast<uint16_t *>(S.blk);
    const int ns = L.ns;
    for (int idx = threadIdx.x; idx < kPage * ns; idx += blockDim.x) {
        const int t = idx / ns, g = idx % ns;
        h[(L.ks >> 1) + kscale_idx(ns, t, g)] = S.kscale[t][g];
        h[(L.km >> 1) + kscale_idx(ns, t, g)] = S.kmin[t][g];
        h[(L.vs >> 1) + vscale_idx(ns, t, g)] = S.vscale[t][g];
        h[(L.vm >> 1) + vscale_idx(ns, t, g)] = S.vmin[t][g];
    }
    for (int t = threadIdx.x; t < kPage; t += blockDim.x) {
        h[(L.k0 >> 1) + k0_idx(t)] = S.kch0[t];
        if (v_ch0) h[(L.v0 >> 1) + t] = S.vch0[t];
    }
}

// Grid: x = work items (sequence, touched page) strided, y = kv head.
// Block: 16 warps.  Each item: read the old block, overwrite the appended
// slots, write it back with 128-bit stores.  T_K[j] is staged once per CTA;
// the transforms of the new rows are spread over all threads (one (slot,
// channel) sum each, four interleaved per thread), then warp w quantizes
// token slot w.  early_release lets a kernel launched after this one with
// programmatic stream serialization start at once (it must not read the
// cache before its own grid-dependency wait).
template <int D, int NS>
__global__ void __launch_bounds__(512) k_quant_pack(
    const float *__restrict__ t_k, const void *__restrict__ kin, const void *__restrict__ vin,
    int dtype, int batch, const int *__restrict__ new_lens, const int *__restrict__ seq_before,
    const int *__restrict__ page_table, int max_pages, int slots_per_seq, uint8_t *__restrict__ pool,
    long long num_pages, int hkv, int v_ch0, int early_release) {
    constexpr int NG = D / kGroup;
    constexpr int kChains = 4;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    AppendSmem<D> &S = *reinterpret_cast<AppendSmem<D> *>(smem_raw);
    const int j = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Layout L = make_layout(D, v_ch0, NS);
    if (early_release) grid_dependents_launch();

    stage_f64_padded<D>(S.tk, t_k + (size_t)j * D * D);
    __syncthreads();

    const int items = batch * slots_per_seq;
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
        const int b = item / slots_per_seq, slot = item % slots_per_seq;
        const int n = new_lens[b], L0 = seq_before[b];
        if (n <= 0) continue;
        const int page = L0 / kPage + slot;
        if (page > (L0 + n - 1) / kPage) continue;
        const int phys = (L0 >= 0 && page < max_pages) ? page_table[(size_t)b * max_pages + page] : -1;
        if (phys < 0 || phys >= num_pages) {
            if (threadIdx.x == 0) dqk_flag_error(kErrBounds);
            continue;
        }
        long long row0 = 0;
        for (int bb = 0; bb < b; ++bb) row0 += new_lens[bb];
        uint4 *blk_g = reinterpret_cast<uint4 *>(pool + ((size_t)phys * hkv + j) * L.bytes);
        // slots [s_lo, s_hi) of this page receive new rows
        const int s_lo = max(0, L0 - page * kPage), s_hi = min(kPage, L0 + n - page * kPage);
        const int total = (s_hi - s_lo) * D;
        const long long row_of_slot = row0 + (long long)page * kPage - L0;   // input row of slot s: + s

        for (int o = threadIdx.x; o < L.bytes / 16; o += blockDim.x) S.blk[o] = blk_g[o];
        for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
            const int sl = s_lo + idx / D, c = idx % D;
            S.x[sl][c] = (double)load_elem(kin, dtype, ((size_t)(row_of_slot + sl) * hkv + j) * D + c);
        }
        __syncthreads();
        unpack_block<D>(S, L, v_ch0);
        // k'_c = sum_i T_K[c][i] x_i, ascending i, exact products summed in fp64
        for (int k0 = threadIdx.x; k0 < total; k0 += kChains * blockDim.x) {
            const double *row[kChains];
            const double *xr[kChains];
            double acc[kChains];
#pragma unroll
            for (int u = 0; u < kChains; ++u) {
                const int k = min(k0 + u * (int)blockDim.x, total - 1);
                const int sl = s_lo + k / D, c = k % D;
                row[u] = &S.tk[c * (D + 1)];
                xr[u] = &S.x[sl][0];
                acc[u] = 0.0;
            }
#pragma unroll 4
            for (int i = 0; i < D; ++i)
#pragma unroll
                for (int u = 0; u < kChains; ++u) acc[u] = fma(row[u][i], xr[u][i], acc[u]);
#pragma unroll
            for (int u = 0; u < kChains; ++u) {
                const int k = k0 + u * (int)blockDim.x;
                if (k < total) S.kp[s_lo + k / D][k % D] = __double2float_rn(acc[u]);
            }
        }
        __syncthreads();
        if (warp >= s_lo && warp < s_hi) {
            float kp[NG];
#pragma unroll
            for (int m = 0; m < NG; ++m) kp[m] = S.kp[warp][lane + 32 * m];
            quantize_warp<NG, NS>(kp, true, lane, S.kcode[warp], S.kscale[warp], S.kmin[warp], &S.kch0[warp]);
            const size_t base = ((size_t)(row_of_slot + warp) * hkv + j) * D;
            float vv[NG];
#pragma unroll
            for (int m = 0; m < NG; ++m) vv[m] = load_elem(vin, dtype, base + lane + 32 * m);
            quantize_warp<NG, NS>(vv, v_ch0 != 0, lane, S.vcode[warp], S.vscale[warp], S.vmin[warp],
                                  &S.vch0[warp]);
        }
        __syncthreads();
        pack_block<D>(S, L, v_ch0);
        __syncthreads();
        for (int o = threadIdx.x; o < L.bytes / 16; o += blockDim.x) blk_g[o] = S.blk[o];
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Row appends of up to a few dozen rows per sequence (decode steps, speculative
// or chunked appends).  D threads (thread c = channel c) handle up to RW
// consecutive new rows of one sequence and kv head: k'_c of every row as
// interleaved independent sums, warp g quantizes group g of each row.  Only
// the rows' own fields of their (page, kv head) blocks are written: key code
// words (each holds codes of one token) with plain stores, value code fields
// (words shared with neighbouring tokens) with atomic and/or, scale/min/
// channel-0 entries with 16-bit stores.  Same arithmetic, hence the same
// bytes, as k_quant_pack.
// ---------------------------------------------------------------------------
constexpr int kDirectMaxNew = 64;   // dqk_append uses k_append_rows up to this many rows per sequence
constexpr int kRowsPerCta = 8;

template <int D, int NS, int RW>
struct RowStoreScratch {
    static constexpr int NG = D / kGroup;
    uint32_t kimg[RW][D], kmask[RW][D], vimg[RW][D], vmask[RW][D];   // code regions: D words each
    float rng[NS == 1 ? RW : 1][4][NG];
};

// Quantize rows i < nr (key k'_c = kp[i], value xv[i] of channel c) at cache
// positions pos0 + i (physical pages phys[i]) and store their fields.  sync()
// synchronises the D threads.
template <int D, int NS, int RW, typename Sync>
__device__ __forceinline__ void quantize_store_rows(const float (&kp)[RW], const float (&xv)[RW], const int (&phys)[RW],
                                                    int nr, int pos0, int c, uint8_t *__restrict__ pool,
                                                    long long num_pages, int hkv, int j, int v_ch0,
                                                    RowStoreScratch<D, NS, RW> &S, Sync sync) {
    constexpr int NG = D / kGroup;
    const int warp = c >> 5, lane = c & 31;
#pragma unroll
    for (int i = 0; i < RW; ++i) {
        S.kimg[i][c] = 0u;
        S.kmask[i][c] = 0u;
        S.vimg[i][c] = 0u;
        S.vmask[i][c] = 0u;
    }
    const Layout L = make_layout(D, v_ch0, NS);
    // group ranges: per warp (32 channels); with one group per row, combined
    // over the row's NG warps through shared memory
    float klo[RW], khi[RW], vlo[RW], vhi[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) {
        // channel 0 keeps its sign; ranges read -0 as +0
        warp_minmax(kp[i] + 0.0f, c == 0, klo[i], khi[i]);
        warp_minmax(xv[i] + 0.0f, v_ch0 != 0 && c == 0, vlo[i], vhi[i]);
        if constexpr (NS == 1) {
            if (lane == 0) {
                S.rng[i][0][warp] = klo[i];
                S.rng[i][1][warp] = khi[i];
                S.rng[i][2][warp] = vlo[i];
                S.rng[i][3][warp] = vhi[i];
            }
        }
    }
    sync();
    if constexpr (NS == 1) {
#pragma unroll
        for (int i = 0; i < RW; ++i)
#pragma unroll
            for (int w = 0; w < NG; ++w) {
                klo[i] = fminf(klo[i], S.rng[i][0][w]);
                khi[i] = fmaxf(khi[i], S.rng[i][1][w]);
                vlo[i] = fminf(vlo[i], S.rng[i][2][w]);
                vhi[i] = fmaxf(vhi[i], S.rng[i][3][w]);
            }
    }
#pragma unroll
    for (int i = 0; i < RW; ++i) {
        if (i >= nr) break;                   // uniform
        if (phys[i] < 0 || phys[i] >= num_pages) {   // uniform
            if (c == 0) dqk_flag_error(kErrBounds);
            continue;
        }
        const int slot = (pos0 + i) % kPage;
        uint16_t *h16 = reinterpret_cast<uint16_t *>(pool + ((size_t)phys[i] * hkv + j) * L.bytes);
        uint16_t ksh, kmh, vsh, vmh;
        const int kc = quant_code(kp[i] + 0.0f, c == 0, klo[i], khi[i], ksh, kmh);
        const int vc = quant_code(xv[i] + 0.0f, v_ch0 != 0 && c == 0, vlo[i], vhi[i], vsh, vmh);
        if (NS == 1 ? c == 0 : lane == 0) {
            const int g = NS == 1 ? 0 : warp;
            h16[(L.ks >> 1) + kscale_idx(NS, slot, g)] = ksh;
            h16[(L.km >> 1) + kscale_idx(NS, slot, g)] = kmh;
            h16[(L.vs >> 1) + vscale_idx(NS, slot, g)] = vsh;
            h16[(L.vm >> 1) + vscale_idx(NS, slot, g)] = vmh;
        }
        if (c == 0) {
            h16[(L.k0 >> 1) + k0_idx(slot)] = f32_to_bf16_rne(kp[i]);
            if (v_ch0) h16[(L.v0 >> 1) + slot] = f32_to_bf16_rne(xv[i]);
        }
        int off, bit;
        kcode_pos(NG, slot, c, off, bit);
        atomicOr(&S.kimg[i][off >> 2], (uint32_t)kc << bit);
        atomicOr(&S.kmask[i][off >> 2], 3u << bit);
        vcode_pos(NG, slot, c, off, bit);
        atomicOr(&S.vimg[i][off >> 2], (uint32_t)vc << bit);
        atomicOr(&S.vmask[i][off >> 2], 3u << bit);
    }
    sync();
#pragma unroll
    for (int i = 0; i < RW; ++i) {
        if (i >= nr) break;
        if (phys[i] < 0 || phys[i] >= num_pages) continue;
        uint8_t *blk = pool + ((size_t)phys[i] * hkv + j) * L.bytes;
        uint32_t *kw = reinterpret_cast<uint32_t *>(blk + L.kc);
        uint32_t *vw = reinterpret_cast<uint32_t *>(blk + L.vc);
        const uint32_t km = S.kmask[i][c], vm = S.vmask[i][c];
        if (km == 0xffffffffu) {
            kw[c] = S.kimg[i][c];             // a key word holds codes of this token only
        } else if (km) {
            atomicAnd(&kw[c], ~km);
            atomicOr(&kw[c], S.kimg[i][c]);
        }
        if (vm) {                             // value words are shared with neighbouring tokens
            atomicAnd(&vw[c], ~vm);
            atomicOr(&vw[c], S.vimg[i][c]);
        }
    }
}

// One CTA of D threads per (group of RW consecutive new rows of a sequence,
// kv head) -- RW = 1 when every sequence appends one row, else kRowsPerCta.
// T_K[j] is staged in shared memory by coalesced 16-byte asynchronous copies
// into rows padded by 16 bytes, so thread c then reads its row c without bank
// conflicts; thread c forms k'_c of every row of the group (fp64 sequential
// sums, the rows i-major in shared memory), then quantize_store_rows.
template <int D, int NS, int RW>
__host__ __device__ constexpr size_t append_rows_smem() {
    return (size_t)D * (D * 4 + 16) + (size_t)RW * D * 8 + sizeof(RowStoreScratch<D, NS, RW>);
}

template <int D, int NS, int RW>
__global__ void __launch_bounds__(D) k_append_rows(
    const float *__restrict__ t_k, const void *__restrict__ kin, const void *__restrict__ vin, int dtype,
    const int *__restrict__ new_lens, const int *__restrict__ seq_before, const int *__restrict__ page_table,
    int max_pages, int groups_per_seq, uint8_t *__restrict__ pool, long long num_pages, int hkv, int v_ch0,
    int early_release) {
    constexpr int kPad = D * 4 + 16;   // bytes per staged row of T_K
    extern __shared__ __align__(16) unsigned char append_rows_mem[];
    unsigned char *sT = append_rows_mem;
    double *xs = reinterpret_cast<double *>(append_rows_mem + (size_t)D * kPad);   // [D][RW], i-major
    RowStoreScratch<D, NS, RW> &S = *reinterpret_cast<RowStoreScratch<D, NS, RW> *>(xs + (size_t)RW * D);
    const int j = blockIdx.y;
    const int b = blockIdx.x / groups_per_seq, t0 = (blockIdx.x - b * groups_per_seq) * RW;
    const int c = threadIdx.x, lane = c & 31;
    if (early_release) grid_dependents_launch();
    const int n = new_lens[b];
    if (t0 >= n) return;   // the whole CTA
    // T_K[j]: D rows of D / 4 chunks, a warp copies 32 consecutive chunks
    {
        const float *tj = t_k + (size_t)j * D * D;
        const uint32_t base = smem_addr(sT);
#pragma unroll 4
        for (int q = c; q < D * D / 4; q += D)
            cp_async16(base + (uint32_t)((q / (D / 4)) * kPad + (q % (D / 4)) * 16), tj + 4 * q);
    }
    const int L0 = seq_before[b];
    int row0 = 0;   // rows of sequences 0..b-1 come first
    for (int bb = lane; bb < b; bb += 32) row0 += new_lens[bb];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) row0 += __shfl_xor_sync(0xffffffffu, row0, o);
    const int nr = min(RW, n - t0);   // rows of this CTA
    float xv[RW];
    int phys[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) {
        const int t = t0 + (i < nr ? i : 0);
        const size_t base = (((size_t)row0 + t) * hkv + j) * D;
        xs[c * RW + i] = (double)load_elem(kin, dtype, base + c);
        xv[i] = load_elem(vin, dtype, base + c);
        const int page = (L0 + t) / kPage;
        phys[i] = (L0 >= 0 && page < max_pages) ? page_table[(size_t)b * max_pages + page] : -1;
    }
    cp_async_wait_all();
    __syncthreads();
    // k'_c = sum_i T_K[c][i] x_i, ascending i, exact products summed in fp64
    double acc[RW];
    {
#pragma unroll
        for (int i = 0; i < RW; ++i) acc[i] = 0.0;
        const unsigned char *row = sT + (size_t)c * kPad;
#pragma unroll 1
        for (int k = 0; k < D / 32; ++k) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float4 tv = *reinterpret_cast<const float4 *>(row + (32 * k + 4 * u) * 4);
                const double t4[4] = {(double)tv.x, (double)tv.y, (double)tv.z, (double)tv.w};
                const double *xi = xs + (32 * k + 4 * u) * RW;
#pragma unroll
                for (int e = 0; e < 4; ++e)
#pragma unroll
                    for (int i = 0; i < RW; ++i) acc[i] = fma(t4[e], xi[e * RW + i], acc[i]);
            }
        }
    }
    float kp[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) kp[i] = __double2float_rn(acc[i]);
    quantize_store_rows<D, NS, RW>(kp, xv, phys, nr, L0 + t0, c, pool, num_pages, hkv, j, v_ch0, S,
                                   [] { __syncthreads(); });
}

}  // namespace dqk
