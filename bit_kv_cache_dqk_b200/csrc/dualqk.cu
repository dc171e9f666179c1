// dualqk.cu -- libdualqk: host side of the C ABI declared in include/dualqk.h
// (argument checks, launch planning) and the single translation unit that
// holds every kernel of the decode hot path.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "append.cuh"
#include "attend.cuh"
#include "bf16.cuh"
#include "decode.cuh"
#include "qprep.cuh"

namespace {

using namespace dqk;

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kMaxDevices = 64;

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

int current_device() {
    int dev = -1;
    return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

int device_sms(int dev) {
    int sms = 0;
    if (dev < 0 || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

// Decode plan and workspace layout: [header | qf | qk | qm | q0 | split
// records], every section 256-byte aligned.
struct DecodePlan {
    int d, G, NT, NG, hc, pps, pw, nchunks, num_ctas, stages, bb, threads, tail;
    size_t off_qf, off_qk, off_qm, off_q0, off_part, bytes, smem;
};

constexpr int kMaxAttendCtas = 160;   // >= the 148 SMs of a B200; larger parts run 160 persistent CTAs

// CTAs of a decode launch: one per SM, but no more than give every CTA about
// three stages of pages when every sequence fills its max_pages: a small
// problem spread over every SM leaves each CTA a stage or less, and each query
// head then has records from dozens of CTAs to merge (several rounds of
// record loads), where a few dozen CTAs stream the same bytes about as fast.
int decode_ctas(int sms, int batch, int nchunks, int max_pages, int pps) {
    const long long units = (long long)batch * nchunks * max_pages;
    const long long per = 3LL * (pps > 0 ? pps : 1);
    const long long want = std::max<long long>(1, (units + per - 1) / per);
    return (int)std::min<long long>(std::min(sms, kMaxAttendCtas), want);
}


size_t records_bytes(size_t runs, int pw, int hc, int G, int d) {
    return ((size_t)kMaxAttendCtas + runs - 1) * pw * hc * G * rec_stride(d) * sizeof(float);
}

size_t prologue_scratch(int d, int ns, int G) {
    if (d == 128) return ns == 1 ? prologue_scratch_bytes<128, 1>(G) : prologue_scratch_bytes<128, 4>(G);
    return ns == 1 ? prologue_scratch_bytes<64, 1>(G) : prologue_scratch_bytes<64, 2>(G);
}

bool plan_decode(const dqk_layer_desc *L, int batch, DecodePlan &P) {
    P.d = L->head_dim;
    P.G = L->num_q_heads / L->num_kv_heads;
    P.NT = P.G > 4 ? 2 : 1;
    P.NG = P.d / kGroup;
    const int hkv = L->num_kv_heads;
    const int warps = attend_warps(P.G), stage_blocks = attend_stage_blocks(P.G);
    P.threads = attend_threads(P.G);
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
    if ((long long)batch * L->num_q_heads >= (1LL << 31) / 2) return false;
    // Records are sized for kMaxAttendCtas so the workspace size does not depend
    // on the device; the launch uses one CTA per SM up to that bound.
    P.num_ctas = kMaxAttendCtas;
    const int ns = P.d / L->group_size;
    P.bb = make_layout(P.d, L->v_ch0_protect, ns).bytes;
    const size_t stage_bytes = (size_t)stage_blocks * P.bb;
    const size_t fixed = decode_fixed_smem(stage_blocks, warps, P.NT, P.NG);
    const size_t budget = 227 * 1024;
    P.stages = (int)std::min<size_t>(kMaxStages, (budget - fixed) / stage_bytes);
    if (P.stages < 2) return false;
    // the shared memory left after the ring (a multiple of 16 bytes) follows
    // it; the prologue works in the last stages and that tail (one stage at
    // least stays free for the producer), the merge in the first stage
    const size_t tail = P.stages == kMaxStages ? 0 : (budget - fixed - P.stages * stage_bytes) & ~(size_t)15;
    P.tail = (int)tail;
    const size_t scratch = prologue_scratch(P.d, ns, P.G);
    const size_t scratch_stages = scratch > tail ? (scratch - tail + stage_bytes - 1) / stage_bytes : 0;
    if (scratch_stages >= (size_t)P.stages) return false;
    if ((size_t)warps * (P.d + 4) * sizeof(float) > stage_bytes) return false;
    P.smem = P.stages * stage_bytes + tail + fixed;
    const size_t R = (size_t)batch * P.nchunks;
    const size_t bj = (size_t)batch * hkv;
    P.off_qf = 256;
    P.off_qk = round_up(P.off_qf + bj * P.NT * P.NG * 32 * sizeof(uint2), 256);
    P.off_qm = round_up(P.off_qk + bj * P.NT * (P.NG + 1) * 4 * sizeof(float), 256);
    P.off_q0 = round_up(P.off_qm + bj * P.NT * 32 * sizeof(uint32_t), 256);
    P.off_part = round_up(P.off_q0 + (size_t)batch * L->num_q_heads * sizeof(float), 256);
    P.bytes = round_up(P.off_part + records_bytes(R, P.pw, P.hc, P.G, P.d), 256);
    return true;
}

dqk_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? DQK_OK : DQK_ERR_CUDA;
}

// Once per (kernel instance, device): the dynamic shared-memory bound, the
// largest carveout (consecutive kernels then do not make the SMs switch their
// L1 / shared split), and a check that one CTA fits on an SM (a cooperative
// launch needs every CTA resident).  Thread-safe; later calls cost a lookup.
template <auto Kernel>
dqk_status prepare_kernel(int dev, size_t smem, int threads) {
    static std::mutex mu;
    static size_t set_smem[kMaxDevices] = {};
    if (dev < 0 || dev >= kMaxDevices) return DQK_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (set_smem[dev] != 0 && set_smem[dev] >= smem) return DQK_OK;
    if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return DQK_ERR_CUDA;
    (void)cudaFuncSetAttribute(Kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, Kernel, threads, smem) != cudaSuccess)
        return DQK_ERR_CUDA;
    if (per_sm < 1) return DQK_ERR_UNSUPPORTED;
    set_smem[dev] = smem;
    return DQK_OK;
}

// The same for kernels launched without a shared-memory bound beyond the
// default: only the carveout.
template <auto Kernel>
void prefer_max_shared(int dev) {
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    if (dev < 0 || dev >= kMaxDevices) return;
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev]) return;
    (void)cudaFuncSetAttribute(Kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    done[dev] = true;
}

// Cooperative launch (every CTA resident: the kernels' grid barriers rely on
// it), with programmatic stream serialization when the device accepts the
// two together: the kernel may then start while the previous kernel of the
// stream finishes; it waits for it (griddepcontrol.wait) before reading
// anything.
std::atomic<int> g_pdl_refused[kMaxDevices];

template <typename... KArgs, typename... Args>
dqk_status launch_cooperative(void (*kernel)(KArgs...), int dev, unsigned grid, unsigned block, size_t smem,
                              cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    const bool pdl = g_pdl_refused[dev].load(std::memory_order_relaxed) == 0;
    cfg.numAttrs = pdl ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
    if (e != cudaSuccess && pdl) {
        (void)cudaGetLastError();   // a refused launch configuration is not sticky
        g_pdl_refused[dev].store(1, std::memory_order_relaxed);
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
    }
    return e == cudaSuccess ? DQK_OK : DQK_ERR_CUDA;
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
    bool partial = false;            // write (m, l, o) records instead of outputs
    // a decode step's append, done inside the kernel (max_new in 1..kFuseMaxNew)
    const void *k = nullptr, *v = nullptr;
    dqk_dtype kv_dtype = DQK_BF16;
    const int *new_lens = nullptr, *seq_before = nullptr;
    int max_new = 0;
    // test only: the producer of CTA 0 never arms its second stage; short ring waits
    bool stall = false;
};

constexpr unsigned long long kRingWaitNs = kWaitLimitNs;   // 1 s
constexpr unsigned long long kGridWaitNs = kWaitLimitNs;
constexpr unsigned long long kStallWaitNs = 1000000ull;     // 1 ms

dqk_status check_decode(const DecodeArgs &a, DecodePlan &P, int &dev) {
    dqk_status st = check_layer(a.L);
    if (st != DQK_OK) return st;
    if (!a.L->t_q || !a.q || !a.seq_lens || !a.page_table || !a.out || !a.ws) return DQK_ERR_INVALID_ARG;
    // the transforms' rows are staged with 16-byte bulk copies
    if (!aligned(a.L->t_q, 16) || (a.max_new > 0 && !aligned(a.L->t_k, 16))) return DQK_ERR_INVALID_ARG;
    if (a.q_dtype != DQK_F32 && a.q_dtype != DQK_BF16) return DQK_ERR_INVALID_ARG;
    if (a.batch <= 0 || a.max_pages <= 0 || a.pct < 0 || a.pct > 99) return DQK_ERR_INVALID_ARG;
    if (!aligned(a.ws, 256) || !aligned(a.out, 16)) return DQK_ERR_INVALID_ARG;
    if (!plan_decode(a.L, a.batch, P)) return DQK_ERR_UNSUPPORTED;
    if (a.ws_bytes < P.bytes) return DQK_ERR_WORKSPACE_TOO_SMALL;
    dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return DQK_ERR_CUDA;
    P.num_ctas = decode_ctas(device_sms(dev), a.batch, P.nchunks, a.max_pages, P.pps);
    if (P.num_ctas <= 0) return DQK_ERR_CUDA;
    return DQK_OK;
}

template <int D, int G, bool VCH0, int NS>
dqk_status run_decode_g(const DecodeArgs &a, const DecodePlan &P, int dev) {
    auto kernel = k_decode<D, G, VCH0, NS>;
    dqk_status st = prepare_kernel<k_decode<D, G, VCH0, NS>>(dev, P.smem, P.threads);
    if (st != DQK_OK) return st;
    char *ws = static_cast<char *>(a.ws);
    DecodeParams dp = {};
    AttendParams &prm = dp.a;
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
    dp.pool_w = static_cast<uint8_t *>(a.L->pool);
    dp.t_q = a.L->t_q;
    dp.q = a.q;
    dp.q_dtype = (int)a.q_dtype;
    dp.pct = a.pct;
    dp.qscale = (float)(1.4426950408889634 / std::sqrt((double)D));
    dp.sel_out = a.sel_out;
    dp.out = a.out;
    dp.partial_out = a.partial ? 1 : 0;
    dp.t_k = a.L->t_k;
    dp.k_in = a.k;
    dp.v_in = a.v;
    dp.kv_dtype = (int)a.kv_dtype;
    dp.max_new = a.max_new;
    dp.new_lens = a.new_lens;
    dp.seq_before = a.seq_before;
    dp.ring_wait_ns = a.stall ? kStallWaitNs : kRingWaitNs;
    dp.grid_wait_ns = kGridWaitNs;
    dp.stall = a.stall ? 1 : 0;
    dp.tail = P.tail;
    return launch_cooperative(kernel, dev, (unsigned)P.num_ctas, (unsigned)P.threads, P.smem, a.stream, dp);
}

template <int D, bool VCH0, int NS>
dqk_status run_decode_s(const DecodeArgs &a, const DecodePlan &P, int dev) {
    switch (P.G) {
        case 1: return run_decode_g<D, 1, VCH0, NS>(a, P, dev);
        case 2: return run_decode_g<D, 2, VCH0, NS>(a, P, dev);
        case 4: return run_decode_g<D, 4, VCH0, NS>(a, P, dev);
        default: return run_decode_g<D, 8, VCH0, NS>(a, P, dev);
    }
}

template <int D, bool VCH0>
dqk_status run_decode_v(const DecodeArgs &a, const DecodePlan &P, int dev) {
    return a.L->group_size == D ? run_decode_s<D, VCH0, 1>(a, P, dev) : run_decode_s<D, VCH0, D / kGroup>(a, P, dev);
}

dqk_status run_decode(const DecodeArgs &a) {
    DecodePlan P;
    int dev = -1;
    dqk_status st = check_decode(a, P, dev);
    if (st != DQK_OK) return st;
    if (a.L->head_dim == 128)
        return a.L->v_ch0_protect ? run_decode_v<128, true>(a, P, dev) : run_decode_v<128, false>(a, P, dev);
    return a.L->v_ch0_protect ? run_decode_v<64, true>(a, P, dev) : run_decode_v<64, false>(a, P, dev);
}

template <int D, int NS>
dqk_status run_append(const dqk_layer_desc *L, const void *k, const void *v, dqk_dtype dtype, int batch,
                      const int *new_lens, const int *seq_before, int max_new, const int *page_table,
                      int max_pages, cudaStream_t stream) {
    const int dev = current_device();
    if (max_new <= kDirectMaxNew) {
        // one row per sequence: one row per CTA, no idle row slots
        const bool one_row = max_new == 1;
        const size_t smem = one_row ? append_rows_smem<D, NS, 1>() : append_rows_smem<D, NS, kRowsPerCta>();
        const dqk_status st = one_row ? prepare_kernel<k_append_rows<D, NS, 1>>(dev, smem, D)
                                      : prepare_kernel<k_append_rows<D, NS, kRowsPerCta>>(dev, smem, D);
        if (st != DQK_OK) return st;
        auto kernel = one_row ? k_append_rows<D, NS, 1> : k_append_rows<D, NS, kRowsPerCta>;
        const int rw = one_row ? 1 : kRowsPerCta;
        const int groups = (max_new + rw - 1) / rw;
        const long long gx = (long long)batch * groups;
        if (gx > 0x7fffffffLL) return DQK_ERR_UNSUPPORTED;
        kernel<<<dim3((unsigned)gx, L->num_kv_heads), D, smem, stream>>>(
            L->t_k, k, v, dtype, new_lens, seq_before, page_table, max_pages, groups,
            static_cast<uint8_t *>(L->pool), L->num_pages, L->num_kv_heads, L->v_ch0_protect, 0);
        return launch_status();
    }
    const size_t smem = sizeof(AppendSmem<D>);
    dqk_status st = prepare_kernel<k_quant_pack<D, NS>>(dev, smem, 512);
    if (st != DQK_OK) return st;
    const int slots = (max_new + kPage - 1) / kPage + 1;
    const long long items = (long long)batch * slots;
    const int sms = std::max(device_sms(dev), 1);
    long long gx = ((long long)sms + L->num_kv_heads - 1) / L->num_kv_heads;   // ~1 CTA per SM (fp64 T_K in smem)
    if (gx > items) gx = items;
    if (gx < 1) gx = 1;
    k_quant_pack<D, NS><<<dim3((unsigned)gx, L->num_kv_heads), 512, smem, stream>>>(
        L->t_k, k, v, dtype, batch, new_lens, seq_before, page_table, max_pages, slots,
        static_cast<uint8_t *>(L->pool), L->num_pages, L->num_kv_heads, L->v_ch0_protect, 0);
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
    if (!aligned(layer->t_k, 16)) return DQK_ERR_INVALID_ARG;
    if (dtype != DQK_F32 && dtype != DQK_BF16) return DQK_ERR_INVALID_ARG;
    if (batch <= 0 || max_pages <= 0 || max_new < 0) return DQK_ERR_INVALID_ARG;
    if (!aligned(k, 4) || !aligned(v, 4)) return DQK_ERR_INVALID_ARG;
    return DQK_OK;
}

dqk_status launch_append(const dqk_layer_desc *layer, const void *k, const void *v, dqk_dtype dtype, int batch,
                         const int *new_lens, const int *seq_lens_before, int max_new, const int *page_table,
                         int max_pages, cudaStream_t s) {
    const bool one = layer->group_size == layer->head_dim;   // one scale group per token
    if (layer->head_dim == 128)
        return one ? run_append<128, 1>(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table,
                                        max_pages, s)
                   : run_append<128, 4>(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table,
                                        max_pages, s);
    return one ? run_append<64, 1>(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table,
                                   max_pages, s)
               : run_append<64, 2>(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table,
                                   max_pages, s);
}
}  // namespace

extern "C" {

dqk_status dqk_append(const dqk_layer_desc *layer, const void *k, const void *v, dqk_dtype dtype, int batch,
                      const int *new_lens, const int *seq_lens_before, int max_new, const int *page_table,
                      int max_pages, dqk_stream_t stream) {
    dqk_status st = check_append(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table, max_pages);
    if (st != DQK_OK || max_new == 0) return st;
    return launch_append(layer, k, v, dtype, batch, new_lens, seq_lens_before, max_new, page_table, max_pages,
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
    return run_decode(a);
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
    int dev = -1;
    st = check_decode(a, P, dev);
    if (st != DQK_OK) return st;
    if (max_new > kFuseMaxNew) {
        // longer appends run as their own kernel first
        st = launch_append(layer, k, v, kv_dtype, batch, new_lens, seq_lens_before, max_new, page_table, max_pages,
                           a.stream);
        if (st != DQK_OK) return st;
    } else if (max_new > 0) {
        a.k = k;
        a.v = v;
        a.kv_dtype = kv_dtype;
        a.new_lens = new_lens;
        a.seq_before = seq_lens_before;
        a.max_new = max_new;
    }
    return run_decode(a);
}

dqk_status dqk_decode_partial(DQK_DECODE_ARGS) {
    DQK_DECODE_PACK;
    a.partial = true;
    return run_decode(a);
}

dqk_status dqk_test_decode_stall(DQK_DECODE_ARGS) {
    DQK_DECODE_PACK;
    a.stall = true;
    return run_decode(a);
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
    return run_decode(a);
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
    P.threads = kB16Threads;
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
    if ((long long)batch * L->num_q_heads >= (1LL << 31) / 2) return false;
    P.num_ctas = kMaxAttendCtas;
    P.bb = b16_block_bytes(P.d);
    const size_t stage_bytes = (size_t)kB16StageBlocks * P.bb;
    const size_t fixed = decode_fixed_smem(kB16StageBlocks, kB16Warps, 1, 0);
    P.stages = (int)std::min<size_t>(kMaxStages, (227 * 1024 - fixed) / stage_bytes);
    if (P.stages < 2) return false;
    if ((size_t)kB16Warps * (P.d + 4) * sizeof(float) > stage_bytes) return false;   // the merge's scratch
    P.smem = P.stages * stage_bytes + fixed;
    const size_t R = (size_t)batch * P.nchunks;
    P.off_qf = P.off_qk = P.off_qm = P.off_q0 = 0;
    P.off_part = 256;
    P.bytes = round_up(P.off_part + records_bytes(R, P.pw, P.hc, P.G, P.d), 256);
    return true;
}

template <int D, int G>
dqk_status run_decode_b16_g(const DecodeArgs &a, const DecodePlan &P, int dev) {
    dqk_status st = prepare_kernel<k_decode_b16<D, G>>(dev, P.smem, P.threads);
    if (st != DQK_OK) return st;
    char *ws = static_cast<char *>(a.ws);
    DecodeParams dp = {};
    AttendParams &prm = dp.a;
    prm.pool = static_cast<const uint8_t *>(a.L->pool);
    prm.num_pages = a.L->num_pages;
    prm.seq_lens = a.seq_lens;
    prm.page_table = a.page_table;
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
    dp.q = a.q;
    dp.q_dtype = (int)a.q_dtype;
    dp.qscale = (float)(1.4426950408889634 / std::sqrt((double)D));
    dp.out = a.out;
    dp.ring_wait_ns = kRingWaitNs;
    dp.grid_wait_ns = kGridWaitNs;
    return launch_cooperative(k_decode_b16<D, G>, dev, (unsigned)P.num_ctas, (unsigned)P.threads, P.smem, a.stream,
                              dp);
}

template <int D>
dqk_status run_decode_b16(const DecodeArgs &a, const DecodePlan &P, int dev) {
    switch (P.G) {
        case 1: return run_decode_b16_g<D, 1>(a, P, dev);
        case 2: return run_decode_b16_g<D, 2>(a, P, dev);
        case 4: return run_decode_b16_g<D, 4>(a, P, dev);
        default: return run_decode_b16_g<D, 8>(a, P, dev);
    }
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
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return DQK_ERR_CUDA;
    P.num_ctas = decode_ctas(device_sms(dev), batch, P.nchunks, max_pages, P.pps);
    if (P.num_ctas <= 0) return DQK_ERR_CUDA;
    DecodeArgs a{layer, q, q_dtype, batch, seq_lens, page_table, max_pages, 0, out, nullptr,
                 workspace, workspace_bytes, static_cast<cudaStream_t>(stream)};
    return layer->head_dim == 128 ? run_decode_b16<128>(a, P, dev) : run_decode_b16<64>(a, P, dev);
}

}  // extern "C"
