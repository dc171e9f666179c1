// dualqk.cu -- libdualqk: host side of the C ABI declared in include/dualqk.h
// (argument checks, launch planning) and the single translation unit that
// holds every kernel of the decode hot path.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "append.cuh"
#include "attend.cuh"
#include "bf16.cuh"
#include "qprep.cuh"

namespace {

using namespace dqk;

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

dqk_status check_layer(const dqk_layer_desc *L) {
    if (!L) return DQK_ERR_INVALID_ARG;
    if (L->head_dim != 64 && L->head_dim != 128) return DQK_ERR_UNSUPPORTED;
    if (L->num_kv_heads <= 0 || L->num_q_heads <= 0 || L->num_q_heads % L->num_kv_heads)
        return DQK_ERR_INVALID_ARG;
    const int G = L->num_q_heads / L->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return DQK_ERR_UNSUPPORTED;
    if (L->page_size != kPage) return DQK_ERR_UNSUPPORTED;
    // scale groups of 32 channels, or one group over the whole head
    if (L->group_size != kGroup && L->group_size != L->head_dim) return DQK_ERR_UNSUPPORTED;
    if (L->v_ch0_protect != 0 && L->v_ch0_protect != 1) return DQK_ERR_INVALID_ARG;
    if (!L->pool || !aligned(L->pool, 16) || L->num_pages <= 0) return DQK_ERR_INVALID_ARG;
    return DQK_OK;
}

int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

// Decode plan and workspace layout: [header | qf | qm | q0 | partial records],
// every section 256-byte aligned.
struct DecodePlan {
    int d, G, NT, NG, hc, pps, pw, nchunks, num_ctas, stages, bb;
    size_t off_qf, off_qk, off_qm, off_q0, off_part, bytes, smem;
};

constexpr int kMaxAttendCtas = 160;   // >= the 148 SMs of a B200; larger parts run 160 persistent CTAs

bool plan_decode(const dqk_layer_desc *L, int batch, DecodePlan &P) {
    P.d = L->head_dim;
    P.G = L->num_q_heads / L->num_kv_heads;
    P.NT = P.G > 4 ? 2 : 1;
    P.NG = P.d / kGroup;
    const int hkv = L->num_kv_heads;
    const int warps = attend_warps(P.G), stage_blocks = attend_stage_blocks(P.G);
    // kv heads per chunk: the largest divisor of Hkv that divides the warp count
    P.hc = 0;
    for (int c = std::min(hkv, warps); c >= 1; --c)
        if (hkv % c == 0 && warps % c == 0) {
            P.hc = c;
            break;
        }
    if (P.hc == 0) return false;
    P.pps = stage_blocks / P.hc;    // pages per stage
    if (P.pps > kMaxPagesPerStage) return false;   // the producer warp fills two page slots per lane
    P.pw = warps / P.hc;            // warps per kv head (each takes attend_pages_per_warp pages of a stage)
    P.nchunks = hkv / P.hc;
    if ((long long)batch * P.nchunks * (L->num_pages + 1) >= (1LL << 31)) return false;
    // Records are sized for kMaxAttendCtas so the workspace size does not depend
    // on the device; the launch (check_decode) uses one CTA per SM up to that bound.
    P.num_ctas = kMaxAttendCtas;
    P.bb = make_layout(P.d, L->v_ch0_protect, P.d / L->group_size).bytes;
    // shared memory: ring stages | mbarriers | valid flags | abort flag | per-warp query fragments
    const size_t stage_bytes = (size_t)stage_blocks * P.bb;
    // (score fragments live in shared memory only for two query-head tiles)
    const size_t fixed = 2 * kMaxStages * sizeof(uint64_t) + (size_t)kMaxStages * stage_blocks + 16 +
                         (P.NT > 1 ? (size_t)warps * P.NT * P.NG * (32 * 8 + 4 * 16) : 0);
    const size_t budget = 227 * 1024;
    P.stages = (int)std::min<size_t>(kMaxStages, (budget - fixed) / stage_bytes);
    if (P.stages < 2) return false;
    P.smem = P.stages * stage_bytes + fixed;
    const size_t R = (size_t)batch * P.nchunks;
    const size_t bj = (size_t)batch * hkv;
    P.off_qf = 256;
    P.off_qk = round_up(P.off_qf + bj * P.NT * P.NG * 32 * sizeof(uint2), 256);
    P.off_qm = round_up(P.off_qk + bj * P.NT * (P.NG + 1) * 4 * sizeof(float), 256);
    P.off_q0 = round_up(P.off_qm + bj * P.NT * 32 * sizeof(uint32_t), 256);
    P.off_part = round_up(P.off_q0 + (size_t)batch * L->num_q_heads * sizeof(float), 256);
    const size_t records = ((size_t)kMaxAttendCtas + R - 1) * P.pw * P.hc * P.G;
    P.bytes = round_up(P.off_part + records * (2 + P.d) * sizeof(float), 256);
    return true;
}

dqk_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? DQK_OK : DQK_ERR_CUDA;
}

struct DecodeArgs {
    const dqk_layer_desc *L;
    const void *q;
    dqk_dtype q_dtype;
    int batch;
    const int *seq_lens, *page_table;
    int max_pages, pct;
    float *out;
    int16_t *sel_out;
    void *ws;
    size_t ws_bytes;
    cudaStream_t stream;
    bool partial = false;      // the combine writes (m, l, o) records instead of outputs
    bool after_append = false; // the query kernel directly follows a step's append (writes first, waits last)
};

dqk_status check_decode(const DecodeArgs &a, DecodePlan &P) {
    dqk_status st = check_layer(a.L);
    if (st != DQK_OK) return st;
    if (!a.L->t_q || !a.q || !a.seq_lens || !a.page_table || !a.out || !a.ws) return DQK_ERR_INVALID_ARG;
    if (a.q_dtype != DQK_F32 && a.q_dtype != DQK_BF16) return DQK_ERR_INVALID_ARG;
    if (a.batch <= 0 || a.max_pages <= 0 || a.pct < 0 || a.pct > 99) return DQK_ERR_INVALID_ARG;
    if (!aligned(a.ws, 256) || !aligned(a.out, 16)) return DQK_ERR_INVALID_ARG;
    if (!plan_decode(a.L, a.batch, P)) return DQK_ERR_UNSUPPORTED;
    if (a.ws_bytes < P.bytes) return DQK_ERR_WORKSPACE_TOO_SMALL;
    P.num_ctas = std::min(device_sms(), kMaxAttendCtas);
    if (P.num_ctas <= 0) return DQK_ERR_CUDA;
    return DQK_OK;
}

// Every kernel of the path prefers the largest shared-memory carveout, so that
// consecutive kernels do not make the SMs switch their L1 / shared split.
// Attributes are per function (one flag per kernel instance); setting one
// twice is harmless.
template <auto Kernel>
void prefer_max_shared() {
    static bool done = false;
    if (!done) {
        (void)cudaFuncSetAttribute(Kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                   (int)cudaSharedmemCarveoutMaxShared);
        done = true;
    }
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream finishes; it orders itself with
// griddepcontrol.wait before touching that kernel's outputs.
template <typename... KArgs, typename... Args>
dqk_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) == cudaSuccess ? DQK_OK : DQK_ERR_CUDA;
}

template <int D>
dqk_status run_prepare(const DecodeArgs &a, const DecodePlan &P) {
    const size_t smem = qprep_smem_bytes(D, P.G);
    prefer_max_shared<k_qprep<D>>();
    if (cudaFuncSetAttribute(k_qprep<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return DQK_ERR_CUDA;
    char *ws = static_cast<char *>(a.ws);
    const float qscale = (float)(1.4426950408889634 / std::sqrt((double)D));
    return launch_pdl(k_qprep<D>, dim3(a.L->num_kv_heads, a.batch), dim3(kQprepThreads), smem, a.stream, a.L->t_q,
                      a.q, (int)a.q_dtype, a.L->num_q_heads, a.L->num_kv_heads, a.pct, qscale,
                      reinterpret_cast<uint2 *>(ws + P.off_qf), reinterpret_cast<float *>(ws + P.off_qk),
                      reinterpret_cast<uint32_t *>(ws + P.off_qm), reinterpret_cast<float *>(ws + P.off_q0),
                      a.sel_out, a.after_append ? 1 : 0);
}

template <int D, int G, bool VCH0, int NS>
dqk_status run_attend_g(const DecodeArgs &a, const DecodePlan &P) {
    prefer_max_shared<k_attend<D, G, VCH0, NS>>();
    if (cudaFuncSetAttribute(k_attend<D, G, VCH0, NS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem) !=
        cudaSuccess)
        return DQK_ERR_CUDA;
    char *ws = static_cast<char *>(a.ws);
    AttendParams prm;
    prm.pool = static_cast<const uint8_t *>(a.L->pool);
    prm.num_pages = a.L->num_pages;
    prm.seq_lens = a.seq_lens;
    prm.page_table = a.page_table;
    prm.qf = reinterpret_cast<const uint2 *>(ws + P.off_qf);
    prm.qk = reinterpret_cast<const float *>(ws + P.off_qk);
    prm.qm = reinterpret_cast<const uint32_t *>(ws + P.off_qm);
    prm.q0 = reinterpret_cast<const float *>(ws + P.off_q0);
    prm.part = reinterpret_cast<float *>(ws + P.off_part);
    prm.batch = a.batch;
    prm.hq = a.L->num_q_heads;
    prm.hkv = a.L->num_kv_heads;
    prm.hc = P.hc;
    prm.pps = P.pps;
    prm.pw = P.pw;
    prm.nchunks = P.nchunks;
    prm.max_pages = a.max_pages;
    prm.bb = P.bb;
    prm.v_ch0 = a.L->v_ch0_protect;
    prm.stages = P.stages;
    prm.num_ctas = P.num_ctas;
    return launch_pdl(k_attend<D, G, VCH0, NS>, dim3(P.num_ctas), dim3(attend_threads(G)), P.smem, a.stream, prm);
}

template <int D, bool VCH0, int NS>
dqk_status run_attend_s(const DecodeArgs &a, const DecodePlan &P) {
    switch (P.G) {
        case 1: return run_attend_g<D, 1, VCH0, NS>(a, P);
        case 2: return run_attend_g<D, 2, VCH0, NS>(a, P);
        case 4: return run_attend_g<D, 4, VCH0, NS>(a, P);
        default: return run_attend_g<D, 8, VCH0, NS>(a, P);
    }
}

template <int D, bool VCH0>
dqk_status run_attend_v(const DecodeArgs &a, const DecodePlan &P) {
    return a.L->group_size == D ? run_attend_s<D, VCH0, 1>(a, P) : run_attend_s<D, VCH0, D / kGroup>(a, P);
}

template <int D>
dqk_status run_attend(const DecodeArgs &a, const DecodePlan &P) {
    return a.L->v_ch0_protect ? run_attend_v<D, true>(a, P) : run_attend_v<D, false>(a, P);
}

template <int D>
dqk_status run_combine(const DecodeArgs &a, const DecodePlan &P) {
    char *ws = static_cast<char *>(a.ws);
    prefer_max_shared<k_combine<D>>();
    return launch_pdl(k_combine<D>, dim3(a.L->num_q_heads, a.batch), dim3(kCombineThreads), 0, a.stream, a.seq_lens,
                      a.batch,
                      a.L->num_q_heads, a.L->num_kv_heads, P.hc, P.pw, P.nchunks, P.num_ctas,
                      reinterpret_cast<const float *>(ws + P.off_part), a.out, (int)a.partial);
}

enum Stage { kPrepare = 1, kAttend = 2, kCombine = 4 };

dqk_status decode_stages(const DecodeArgs &a, int stages) {
    DecodePlan P;
    dqk_status st = check_decode(a, P);
    if (st != DQK_OK) return st;
    const bool d128 = a.L->head_dim == 128;
    if (stages & kPrepare) {
        st = d128 ? run_prepare<128>(a, P) : run_prepare<64>(a, P);
        if (st != DQK_OK) return st;
    }
    if (stages & kAttend) {
        st = d128 ? run_attend<128>(a, P) : run_attend<64>(a, P);
        if (st != DQK_OK) return st;
    }
    if (stages & kCombine) {
        st = d128 ? run_combine<128>(a, P) : run_combine<64>(a, P);
        if (st != DQK_OK) return st;
    }
    return DQK_OK;
}

template <int D, int NS>
dqk_status run_append(const dqk_layer_desc *L, const void *k, const void *v, dqk_dtype dtype, int batch,
                      const int *new_lens, const int *seq_before, int max_new, const int *page_table,
                      int max_pages, int early_release, cudaStream_t stream) {
    if (max_new <= kDirectMaxNew) {
        // one row per sequence (a decode step): one row per CTA, no idle row slots
        if (max_new == 1) prefer_max_shared<k_append_rows<D, NS, 1>>();
        else prefer_max_shared<k_append_rows<D, NS, kRowsPerCta>>();
        auto kernel = max_new == 1 ? k_append_rows<D, NS, 1> : k_append_rows<D, NS, kRowsPerCta>;
        const int rw = max_new == 1 ? 1 : kRowsPerCta;
        const int groups = (max_new + rw - 1) / rw;
        const long long gx = (long long)batch * groups;
        if (gx > 0x7fffffffLL) return DQK_ERR_UNSUPPORTED;
        kernel<<<dim3((unsigned)gx, L->num_kv_heads), D, 0, stream>>>(
            L->t_k, k, v, dtype, new_lens, seq_before, page_table, max_pages, groups,
            static_cast<uint8_t *>(L->pool), L->num_pages, L->num_kv_heads, L->v_ch0_protect, early_release);
        return launch_status();
    }
    const size_t smem = sizeof(AppendSmem<D>);
    if (cudaFuncSetAttribute(k_quant_pack<D, NS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return DQK_ERR_CUDA;
    const int slots = (max_new + kPage - 1) / kPage + 1;
    const long long items = (long long)batch * slots;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long gx = ((long long)sms + L->num_kv_heads - 1) / L->num_kv_heads;   // ~1 CTA per SM (fp64 T_K in smem)
    if (gx > items) gx = items;
    if (gx < 1) gx = 1;
    k_quant_pack<D, NS><<<dim3((unsigned)gx, L->num_kv_heads), 512, smem, stream>>>(
        L->t_k, k, v, dtype, batch, new_lens, seq_before, page_table, max_pages, slots,
        static_cast<uint8_t *>(L->pool), L->num_pages, L->num_kv_heads, L->v_ch0_protect, early_release);
    return launch_status();
}

}  // namespace

extern "C" {

size_t dqk_block_bytes(const dqk_layer_desc *layer) {
    if (!layer || (layer->head_dim != 64 && layer->head_dim != 128)) return 0;
    if (layer->v_ch0_protect != 0 && layer->v_ch0_protect != 1) return 0;
    if (layer->group_size != kGroup && layer->group_size != layer->head_dim) return 0;
    return (size_t)make_layout(layer->head_dim, layer->v_ch0_protect, layer->head_dim / layer->group_size).bytes;
}

}  // extern "C"

namespace {
dqk_status check_append(const dqk_layer_desc *layer, const void *k, const void *v, dqk_dtype dtype, int batch,
                        const int *new_lens, const int *seq_lens_before, int max_new, const int *page_table,
                        int max_pages) {
    dqk_status st = check_layer(layer);
    if (st != DQK_OK) return st;
    if (!layer->t_k || !k || !v || !new_lens || !seq_lens_before || !page_table) return DQK_ERR_INVALID_ARG;
    if (dtype != DQK_F32 && dtype != DQK_BF16) return DQK_ERR_INVALID_ARG;
    if (batch <= 0 || max_pages <= 0 || max_new < 0) return DQK_ERR_INVALID_ARG;
    if (!aligned(k, 4) || !aligned(v, 4)) return DQK_ERR_INVALID_ARG;
    return DQK_OK;
}

dqk_status launch_append(const dqk_layer_desc *layer, const void *k, const void *v, dqk_dtype dtype, int batch,
                         const int *new_lens, const int *seq_lens_before, int max_new, const int *page_table,
                         int max_pages, int early_release, cudaStream_t s) {
    const bool one = layer->group_size == layer->head_dim;   // one scale group per token
    if (layer->head_dim == 128)
        return one ? run_append<128, 1>(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table,
                                        max_pages, early_release, s)
                   : run_append<128, 4>(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table,
                                        max_pages, early_release, s);
    return one ? run_append<64, 1>(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table,
                                   max_pages, early_release, s)
               : run_append<64, 2>(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table,
                                   max_pages, early_release, s);
}
}  // namespace

extern "C" {

dqk_status dqk_append(const dqk_layer_desc *layer, const void *k, const void *v, dqk_dtype dtype, int batch,
                      const int *new_lens, const int *seq_lens_before, int max_new, const int *page_table,
                      int max_pages, dqk_stream_t stream) {
    dqk_status st = check_append(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table, max_pages);
    if (st != DQK_OK || max_new == 0) return st;
    // whatever follows may read the cache at once: release it only at exit
    return launch_append(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table, max_pages, 0,
                         static_cast<cudaStream_t>(stream));
}

size_t dqk_decode_workspace_size(const dqk_layer_desc *layer, int batch, int max_pages) {
    if (check_layer(layer) != DQK_OK || batch <= 0 || max_pages <= 0) return 0;
    DecodePlan P;
    if (!plan_decode(layer, batch, P)) return 0;
    return P.bytes;
}

#define DQK_DECODE_ARGS                                                                                   \
    const dqk_layer_desc *layer, const void *q, dqk_dtype q_dtype, int batch, const int *seq_lens,        \
        const int *page_table, int max_pages, int sparsity_pct, float *out, int16_t *sel_out, void *workspace, \
        size_t workspace_bytes, dqk_stream_t stream
#define DQK_DECODE_PACK                                                                                   \
    DecodeArgs a{layer, q, q_dtype, batch, seq_lens, page_table, max_pages, sparsity_pct, out, sel_out,   \
                 workspace, workspace_bytes, static_cast<cudaStream_t>(stream)}

dqk_status dqk_decode(DQK_DECODE_ARGS) {
    DQK_DECODE_PACK;
    return decode_stages(a, kPrepare | kAttend | kCombine);
}
dqk_status dqk_decode_step(const dqk_layer_desc *layer, const void *k, const void *v, dqk_dtype kv_dtype,
                           const int *new_lens, const int *seq_lens_before, int max_new, const void *q,
                           dqk_dtype q_dtype, int batch, const int *seq_lens, const int *page_table, int max_pages,
                           int sparsity_pct, float *out, int16_t *sel_out, void *workspace, size_t workspace_bytes,
                           dqk_stream_t stream) {
    dqk_status st = check_append(layer, k, v, kv_dtype, batch, new_lens, seq_lens_before, max_new, page_table,
                                 max_pages);
    if (st != DQK_OK) return st;
    DecodeArgs a{layer, q, q_dtype, batch, seq_lens, page_table, max_pages, sparsity_pct, out, sel_out,
                 workspace, workspace_bytes, static_cast<cudaStream_t>(stream)};
    DecodePlan P;
    st = check_decode(a, P);
    if (st != DQK_OK) return st;
    if (max_new > 0) {
        // the query kernel (next on the stream) may start at once: it reads only
        // q and T_Q before its grid-dependency wait
        st = launch_append(layer, k, v, kv_dtype, batch, new_lens, seq_lens_before, max_new, page_table, max_pages,
                           1, a.stream);
        if (st != DQK_OK) return st;
        a.after_append = true;
    }
    return decode_stages(a, kPrepare | kAttend | kCombine);
}
dqk_status dqk_decode_partial(DQK_DECODE_ARGS) {
    DQK_DECODE_PACK;
    a.partial = true;
    return decode_stages(a, kPrepare | kAttend | kCombine);
}

dqk_status dqk_merge_partials(const float *parts, int n_parts, int batch, int num_q_heads, int head_dim,
                              float *out, dqk_stream_t stream) {
    if (!parts || !out || n_parts <= 0 || batch <= 0 || num_q_heads <= 0) return DQK_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return DQK_ERR_UNSUPPORTED;
    if (!aligned(parts, 4) || !aligned(out, 4)) return DQK_ERR_INVALID_ARG;
    const long long rows = (long long)batch * num_q_heads;
    if (rows > 0x7fffffffLL) return DQK_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (head_dim == 128)
        k_merge<128><<<(unsigned)rows, 128, 0, s>>>(parts, n_parts, rows, out);
    else
        k_merge<64><<<(unsigned)rows, 64, 0, s>>>(parts, n_parts, rows, out);
    return launch_status();
}

dqk_status dqk_decode_prepare(DQK_DECODE_ARGS) {
    DQK_DECODE_PACK;
    return decode_stages(a, kPrepare);
}
dqk_status dqk_decode_attend(DQK_DECODE_ARGS) {
    DQK_DECODE_PACK;
    return decode_stages(a, kAttend);
}
dqk_status dqk_decode_combine(DQK_DECODE_ARGS) {
    DQK_DECODE_PACK;
    return decode_stages(a, kCombine);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// dqk_decode_noalloc: the decode for callers that cannot hand over a device
// workspace.  Its scratch is this file-scope array in the module's static
// device memory (one per device that loads the library).  Host code must not
// pass the symbol itself to a kernel -- on the host it is only a stand-in --
// so its device address is looked up with cudaGetSymbolAddress, once per
// device, on that device's first call.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_dqk_noalloc_ws[DQK_NOALLOC_WORKSPACE_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

dqk_status noalloc_workspace(void **ws) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DQK_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return DQK_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dqk_noalloc_ws) != cudaSuccess || !p) return DQK_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *ws = g_noalloc_ptr[dev];
    return DQK_OK;
}
}  // namespace

extern "C" {

dqk_status dqk_decode_noalloc(const dqk_layer_desc *layer, const void *q, dqk_dtype q_dtype, int batch,
                              const int *seq_lens, const int *page_table, int max_pages, int sparsity_pct,
                              float *out, int16_t *sel_out, dqk_stream_t stream) {
    dqk_status st = check_layer(layer);
    if (st != DQK_OK) return st;
    if (batch <= 0 || max_pages <= 0) return DQK_ERR_INVALID_ARG;
    DecodePlan P;
    if (!plan_decode(layer, batch, P)) return DQK_ERR_UNSUPPORTED;
    if (P.bytes > (size_t)DQK_NOALLOC_WORKSPACE_BYTES) return DQK_ERR_WORKSPACE_TOO_SMALL;
    void *ws = nullptr;
    st = noalloc_workspace(&ws);
    if (st != DQK_OK) return st;
    DecodeArgs a{layer, q, q_dtype, batch, seq_lens, page_table, max_pages, sparsity_pct, out, sel_out,
                 ws, (size_t)DQK_NOALLOC_WORKSPACE_BYTES, static_cast<cudaStream_t>(stream)};
    return decode_stages(a, kPrepare | kAttend | kCombine);
}

dqk_status dqk_last_device_error(dqk_stream_t stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DQK_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_dqk_device_error, sizeof(word)) != cudaSuccess) return DQK_ERR_CUDA;
    if (word && cudaMemcpyToSymbol(g_dqk_device_error, &zero, sizeof(zero)) != cudaSuccess) return DQK_ERR_CUDA;
    if (word & kErrBounds) return DQK_ERR_DEVICE_BOUNDS;
    if (word & kErrTimeout) return DQK_ERR_TIMEOUT;
    return DQK_OK;
}

const char *dqk_status_string(dqk_status s) {
    switch (s) {
        case DQK_OK: return "DQK_OK";
        case DQK_ERR_INVALID_ARG: return "DQK_ERR_INVALID_ARG";
        case DQK_ERR_UNSUPPORTED: return "DQK_ERR_UNSUPPORTED";
        case DQK_ERR_WORKSPACE_TOO_SMALL: return "DQK_ERR_WORKSPACE_TOO_SMALL";
        case DQK_ERR_CUDA: return "DQK_ERR_CUDA";
        case DQK_ERR_DEVICE_BOUNDS: return "DQK_ERR_DEVICE_BOUNDS";
        case DQK_ERR_TIMEOUT: return "DQK_ERR_TIMEOUT";
    }
    return "DQK_UNKNOWN_STATUS";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// The BF16 comparison decode (paged BF16 cache, no transform / quantization /
// pruning): append, workspace size, decode.
// ---------------------------------------------------------------------------
namespace {

dqk_status check_layer_b16(const dqk_layer_desc *L) {
    if (!L) return DQK_ERR_INVALID_ARG;
    if (L->head_dim != 64 && L->head_dim != 128) return DQK_ERR_UNSUPPORTED;
    if (L->num_kv_heads <= 0 || L->num_q_heads <= 0 || L->num_q_heads % L->num_kv_heads)
        return DQK_ERR_INVALID_ARG;
    const int G = L->num_q_heads / L->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return DQK_ERR_UNSUPPORTED;
    if (L->page_size != kPage) return DQK_ERR_UNSUPPORTED;
    if (!L->pool || !aligned(L->pool, 16) || L->num_pages <= 0) return DQK_ERR_INVALID_ARG;
    return DQK_OK;
}

bool plan_b16(const dqk_layer_desc *L, int batch, DecodePlan &P) {
    P.d = L->head_dim;
    P.G = L->num_q_heads / L->num_kv_heads;
    P.NT = P.G > 4 ? 2 : 1;
    P.NG = P.d / kGroup;
    const int hkv = L->num_kv_heads;
    if (hkv <= kB16Warps) {
        if (kB16Warps % hkv) return false;
        P.hc = hkv;
    } else {
        if (hkv % kB16Warps) return false;
        P.hc = kB16Warps;
    }
    P.pps = kB16StageBlocks / P.hc;
    P.pw = kB16Warps / P.hc;
    P.nchunks = hkv / P.hc;
    if ((long long)batch * P.nchunks * (L->num_pages + 1) >= (1LL << 31)) return false;
    P.num_ctas = kMaxAttendCtas;
    P.bb = b16_block_bytes(P.d);
    const size_t stage_bytes = (size_t)kB16StageBlocks * P.bb;
    const size_t fixed = 2 * kMaxStages * sizeof(uint64_t) + (size_t)kMaxStages * kB16StageBlocks + 16;
    P.stages = (int)std::min<size_t>(kMaxStages, (227 * 1024 - fixed) / stage_bytes);
    if (P.stages < 2) return false;
    P.smem = P.stages * stage_bytes + fixed;
    const size_t R = (size_t)batch * P.nchunks;
    const size_t bj = (size_t)batch * hkv;
    P.off_qf = 256;
    P.off_qk = P.off_qm = P.off_q0 = 0;
    P.off_part = round_up(P.off_qf + bj * P.NT * (P.d / 16) * 32 * sizeof(uint2), 256);
    const size_t records = ((size_t)kMaxAttendCtas + R - 1) * P.pw * P.hc * P.G;
    P.bytes = round_up(P.off_part + records * (2 + P.d) * sizeof(float), 256);
    return true;
}

template <int D, int G>
dqk_status run_attend_b16(const DecodeArgs &a, const DecodePlan &P) {
    if (cudaFuncSetAttribute(k_attend_b16<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem) !=
        cudaSuccess)
        return DQK_ERR_CUDA;
    char *ws = static_cast<char *>(a.ws);
    AttendParams prm = {};
    prm.pool = static_cast<const uint8_t *>(a.L->pool);
    prm.num_pages = a.L->num_pages;
    prm.seq_lens = a.seq_lens;
    prm.page_table = a.page_table;
    prm.qf = reinterpret_cast<const uint2 *>(ws + P.off_qf);
    prm.part = reinterpret_cast<float *>(ws + P.off_part);
    prm.batch = a.batch;
    prm.hq = a.L->num_q_heads;
    prm.hkv = a.L->num_kv_heads;
    prm.hc = P.hc;
    prm.pps = P.pps;
    prm.pw = P.pw;
    prm.nchunks = P.nchunks;
    prm.max_pages = a.max_pages;
    prm.bb = P.bb;
    prm.v_ch0 = 0;
    prm.stages = P.stages;
    prm.num_ctas = P.num_ctas;
    return launch_pdl(k_attend_b16<D, G>, dim3(P.num_ctas), dim3(kB16Threads), P.smem, a.stream, prm);
}

template <int D>
dqk_status run_decode_b16(const DecodeArgs &a, const DecodePlan &P) {
    char *ws = static_cast<char *>(a.ws);
    const float qscale = (float)(1.4426950408889634 / std::sqrt((double)D));
    k_qprep_b16<D><<<dim3(a.L->num_kv_heads, a.batch), 128, 0, a.stream>>>(
        a.q, (int)a.q_dtype, a.L->num_q_heads, a.L->num_kv_heads, qscale, reinterpret_cast<uint2 *>(ws + P.off_qf));
    dqk_status st = launch_status();
    if (st != DQK_OK) return st;
    switch (P.G) {
        case 1: st = run_attend_b16<D, 1>(a, P); break;
        case 2: st = run_attend_b16<D, 2>(a, P); break;
        case 4: st = run_attend_b16<D, 4>(a, P); break;
        default: st = run_attend_b16<D, 8>(a, P); break;
    }
    if (st != DQK_OK) return st;
    return run_combine<D>(a, P);
}

}  // namespace

extern "C" {

size_t dqk_bf16_block_bytes(const dqk_layer_desc *layer) {
    if (!layer || (layer->head_dim != 64 && layer->head_dim != 128)) return 0;
    return (size_t)b16_block_bytes(layer->head_dim);
}

dqk_status dqk_bf16_append(const dqk_layer_desc *layer, const void *k, const void *v, dqk_dtype dtype, int batch,
                           const int *new_lens, const int *seq_lens_before, int max_new, const int *page_table,
                           int max_pages, dqk_stream_t stream) {
    dqk_status st = check_layer_b16(layer);
    if (st != DQK_OK) return st;
    if (!k || !v || !new_lens || !seq_lens_before || !page_table) return DQK_ERR_INVALID_ARG;
    if (dtype != DQK_F32 && dtype != DQK_BF16) return DQK_ERR_INVALID_ARG;
    if (batch <= 0 || max_pages <= 0 || max_new < 0) return DQK_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(v, 16)) return DQK_ERR_INVALID_ARG;
    if (max_new == 0) return DQK_OK;
    const long long gx = (long long)batch * max_new;
    if (gx > 0x7fffffffLL) return DQK_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *pool = static_cast<uint8_t *>(layer->pool);
    if (layer->head_dim == 128)
        k_append_b16<128><<<dim3((unsigned)gx, layer->num_kv_heads), 2 * 128 / 8, 0, s>>>(
            k, v, dtype, new_lens, seq_lens_before, page_table, max_pages, max_new, pool, layer->num_pages,
            layer->num_kv_heads);
    else
        k_append_b16<64><<<dim3((unsigned)gx, layer->num_kv_heads), 2 * 64 / 8, 0, s>>>(
            k, v, dtype, new_lens, seq_lens_before, page_table, max_pages, max_new, pool, layer->num_pages,
            layer->num_kv_heads);
    return launch_status();
}

size_t dqk_bf16_decode_workspace_size(const dqk_layer_desc *layer, int batch, int max_pages) {
    if (check_layer_b16(layer) != DQK_OK || batch <= 0 || max_pages <= 0) return 0;
    DecodePlan P;
    if (!plan_b16(layer, batch, P)) return 0;
    return P.bytes;
}

dqk_status dqk_bf16_decode(const dqk_layer_desc *layer, const void *q, dqk_dtype q_dtype, int batch,
                           const int *seq_lens, const int *page_table, int max_pages, float *out, void *workspace,
                           size_t workspace_bytes, dqk_stream_t stream) {
    dqk_status st = check_layer_b16(layer);
    if (st != DQK_OK) return st;
    if (!q || !seq_lens || !page_table || !out || !workspace) return DQK_ERR_INVALID_ARG;
    if (q_dtype != DQK_F32 && q_dtype != DQK_BF16) return DQK_ERR_INVALID_ARG;
    if (batch <= 0 || max_pages <= 0) return DQK_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || !aligned(out, 16)) return DQK_ERR_INVALID_ARG;
    DecodePlan P;
    if (!plan_b16(layer, batch, P)) return DQK_ERR_UNSUPPORTED;
    if (workspace_bytes < P.bytes) return DQK_ERR_WORKSPACE_TOO_SMALL;
    P.num_ctas = std::min(device_sms(), kMaxAttendCtas);
    if (P.num_ctas <= 0) return DQK_ERR_CUDA;
    DecodeArgs a{layer, q, q_dtype, batch, seq_lens, page_table, max_pages, 0, out, nullptr,
                 workspace, workspace_bytes, static_cast<cudaStream_t>(stream)};
    return layer->head_dim == 128 ? run_decode_b16<128>(a, P) : run_decode_b16<64>(a, P);
}

}  // extern "C"
