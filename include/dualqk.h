/*
 * dualqk.h -- C ABI of libdualqk, the B200 (sm_100a) decode hot path of
 * Dual-QK: paired key/query transforms, INT2 KV cache with BF16 key channel 0,
 * and query-channel-pruned attention over a paged cache.
 *
 * What the method is (page titles and sections):
 *  - "How does Dual-QK compress KV caches to 2-bit while keeping accuracy at
 *    128K context?", section "Paired transforms instead of shared rotation":
 *    a non-orthogonal key transform T_K (partial key whitening) flattens keys
 *    for INT2 storage, a paired query transform T_Q (query-aligned basis)
 *    sharpens queries for channel pruning, channel 0 is protected.
 *  - same page, section "Why the cache becomes a bottleneck": the pair must
 *    preserve query-key dot products, so T_Q = T_K^{-T} and (T_Q q).(T_K k)
 *    = q.k; query-channel pruning reduces key-cache reads.
 *  - same page, section "Throughput on SGLang": 2 bits per stored value and
 *    40 % of key channels removed from reads.
 *  - "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches",
 *    abstract: INT2 K/V, channel-0 protection, 40 % query-channel sparsity.
 * Details the pages leave open are fixed as follows: asymmetric INT2 per token
 * in groups of 32 channels with fp16 scale and min, codes rounded half to even,
 * top-k ties broken toward the lower channel index, RoPE applied by the caller
 * before T_K, key channel 0 in BF16 (value channel 0 optionally).
 *
 * Conventions for every call:
 *  - Ownership: the caller allocates and owns every buffer (pool, page tables,
 *    q/k/v, out, workspace).  The library allocates nothing and keeps no state
 *    besides one device error word per device (see dqk_last_device_error) and
 *    the static scratch of dqk_decode_noalloc.
 *  - Pointers marked (device) must be device memory of the current device;
 *    (host) means host memory.  All work is enqueued on `stream` (a
 *    cudaStream_t value, NULL for the legacy default stream); no call
 *    synchronizes except dqk_last_device_error.
 *  - Errors: every call returns a dqk_status.  Invalid arguments are rejected
 *    before anything is launched.  A failed launch returns DQK_ERR_CUDA.
 *    Out-of-range page ids or lengths found on the device do not fault: the
 *    kernel skips the access and sets the device error word.
 */
#ifndef DUALQK_H
#define DUALQK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void *dqk_stream_t; /* a cudaStream_t */

typedef enum {
    DQK_OK = 0,
    DQK_ERR_INVALID_ARG = 1,         /* null pointer, bad size, bad layer descriptor */
    DQK_ERR_UNSUPPORTED = 2,         /* head_dim, group ratio or page size not built */
    DQK_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes < dqk_decode_workspace_size */
    DQK_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
    DQK_ERR_DEVICE_BOUNDS = 5,       /* device saw a page id / length out of range */
    DQK_ERR_TIMEOUT = 6              /* a bounded device wait gave up */
} dqk_status;

typedef enum { DQK_F32 = 0, DQK_BF16 = 1 } dqk_dtype;

/* One attention layer's cache description.
 *  head_dim       64 or 128 (d).
 *  num_q_heads    Hq; num_kv_heads Hkv; Hq % Hkv == 0 and G = Hq/Hkv in
 *                 {1, 2, 4, 8}.  Query head h reads kv head h / G.
 *  page_size      must be 16 tokens.
 *  group_size     channels per (scale, min) group: 32, or head_dim for one
 *                 group per token (74 B per token and kv head at d = 128,
 *                 the compression "Results at 128K context" reports).
 *  v_ch0_protect  0: value channel 0 quantized like the others (default);
 *                 1: value channel 0 kept in BF16 as well.
 *  t_k, t_q       (device) fp32 [Hkv][d][d] row-major: k' = T_K k,
 *                 q' = T_Q q.  The caller supplies T_Q = T_K^{-T}.  16-byte
 *                 aligned (DQK_ERR_INVALID_ARG otherwise).
 *  pool           (device) the paged cache: num_pages * Hkv blocks of
 *                 dqk_block_bytes() bytes, block (page p, kv head j) at byte
 *                 offset (p * Hkv + j) * dqk_block_bytes().  16-byte aligned.
 */
typedef struct {
    int head_dim;
    int num_q_heads;
    int num_kv_heads;
    int page_size;
    int group_size;
    int v_ch0_protect;
    const float *t_k;
    const float *t_q;
    void *pool;
    long long num_pages;
} dqk_layer_desc;

/* Bytes of one (page, kv head) block: 16 tokens of INT2 codes, fp16
 * scale/min per group for K and V, and the BF16 channel 0.  Groups of 32:
 * d = 128: 1568 (98 B per token and kv head), d = 64: 800 (50 B); one group
 * per token: 1184 (74 B) and 672 (42 B); +32 with v_ch0_protect.  Returns 0
 * for an unsupported descriptor.
 *
 * Block layout (byte offsets, NG = d/32 code blocks, NS = d/group_size scale
 * groups, P = 16 tokens; the code sections are in the operand order of the
 * decode kernel's tensor-core tiles, each lane of a warp reading 4*NG
 * contiguous bytes):
 *   KC = 0            K codes, 4*d bytes: code of (token t, channel c) is in the
 *                     32-bit word at KC + 4*(lane*NG + W), bit 8*j + 2*f, with
 *                     g=c/32, cc=c%32, r=2*(cc/16)+t/8, lane=4*(t%8)+(cc%16)/4,
 *                     j=cc%4, W=r%NG, f=g+NG*(r/NG).
 *   KS = 4d           K scale fp16 [t][g], g < NS
 *   KM = KS + 32*NS   K min   fp16 [t][g]
 *   K0 = KM + 32*NS   K channel 0 BF16, token t at index 2*(t%8) + t/8
 *   VC = K0 + 32      V codes, 4*d bytes: (t, c) is in the word at
 *                     VC + 4*(lane*NG + W), bit 16*e + 2*i, with m=c/16,
 *                     cr=(c%16)/8, tb=t/8, tig=(t%8)/2, e=t%2,
 *                     lane=4*(c%8)+tig; NG=4: W=cr+2*tb, i=m;
 *                     NG=2: q=(2m+cr)*2+tb, W=q/8, i=q%8.
 *   VS = VC + 4d      V scale fp16, (t, g) at index 2*(NS*(t/2) + g) + t%2
 *   VM = VS + 32*NS   V min fp16, same indexing
 *   V0 = VM + 32*NS   V channel 0 BF16 [t] (only with v_ch0_protect)
 * The code slot of a protected channel 0 holds 0.
 */
size_t dqk_block_bytes(const dqk_layer_desc *layer);

/* dqk_append -- transform, quantize and pack new K/V rows into the cache.
 * Passages: key transform and INT2 storage with channel-0 protection ("Paired
 * transforms instead of shared rotation"; "Throughput on SGLang").
 *  k, v             (device) [sum(new_lens)][Hkv][d] rows, dtype DQK_F32 or
 *                   DQK_BF16, sequence b's rows after those of b-1; RoPE
 *                   already applied to k.
 *  new_lens         (device) int [batch]: rows appended to sequence b.
 *  seq_lens_before  (device) int [batch]: tokens already cached; the rows go
 *                   to positions seq_lens_before[b] .. +new_lens[b]-1.
 *  max_new          (host) upper bound of new_lens[] (sizes the launch).
 *  page_table       (device) int [batch][max_pages]: logical page -> physical
 *                   page in the pool; entries covering the new positions must
 *                   be valid and not shared with another sequence being
 *                   appended in the same call.
 * Per token and kv head: k' = fp32(fp64 sum over i ascending of
 * T_K[c][i]*k[i]); per group g (group_size channels): scale =
 * fp16((max-min)/3), min = fp16(min)
 * (fp64 arithmetic, RNE, saturating), code = clamp(rne((x-min)/scale), 0, 3)
 * or 0 when scale == 0; key channel 0 -> BF16, left out of group 0's range.
 * Values: same quantizer, no transform.  Positions of the touched pages that
 * are not appended keep their bytes.  The caller advances its lengths.
 */
dqk_status dqk_append(const dqk_layer_desc *layer, const void *k, const void *v, dqk_dtype dtype,
                      int batch, const int *new_lens, const int *seq_lens_before, int max_new,
                      const int *page_table, int max_pages, dqk_stream_t stream);

/* Device workspace needed by dqk_decode for `batch` sequences of at most
 * max_pages pages (query prep, split partials, counters).  0 = unsupported. */
size_t dqk_decode_workspace_size(const dqk_layer_desc *layer, int batch, int max_pages);

/* dqk_decode -- pruned-channel attention of one decode query per head.
 * Passages: channel pruning of the query ("Why the cache becomes a
 * bottleneck"; "Throughput on SGLang": 40 % of key channels removed from
 * reads), attention over the INT2 cache.
 *  q            (device) [batch][Hq][d], DQK_F32 or DQK_BF16, RoPE applied.
 *  seq_lens     (device) int [batch]: tokens to attend (appended ones
 *               included); 0 gives a zero output row.
 *  page_table   (device) int [batch][max_pages].
 *  sparsity_pct 0..99: n_keep = d - floor(pct*d/100) channels are kept per
 *               query head, channel 0 always, then the largest |q'_c| of
 *               channels 1..d-1, ties to the lower index.
 *  out          (device) fp32 [batch][Hq][d].
 *  sel_out      (device, nullable) int16 [batch][Hq][n_keep]: the kept
 *               channels in ascending order.
 *  workspace    (device) >= dqk_decode_workspace_size(layer, batch,
 *               max_pages) bytes, 256-byte aligned; contents need no
 *               initialisation and are scratch after the call.
 * q' = fp32(fp64 sequential T_Q q); s_t = q'_S . k^'_t / sqrt(d) over the
 * kept channels with k^' = min + code*scale (BF16 value for channel 0);
 * out = softmax(s) . v^.  Computed as split-K flash decoding in one
 * cooperative kernel launch (one CTA per SM): the query transform and
 * selection of every head spread over the CTAs, a grid barrier, the online
 * softmax over each CTA's share of the pages with fp32 partials (m, l, o),
 * a second grid barrier, then the log-sum-exp merge of each head's
 * partials.  The kernel is launched with programmatic stream serialization
 * where the device accepts it together with the cooperative attribute; it
 * waits for the previous kernel of the stream before reading anything.
 */
dqk_status dqk_decode(const dqk_layer_desc *layer, const void *q, dqk_dtype q_dtype, int batch,
                      const int *seq_lens, const int *page_table, int max_pages,
                      int sparsity_pct, float *out, int16_t *sel_out, void *workspace,
                      size_t workspace_bytes, dqk_stream_t stream);

/* dqk_decode_step -- one serving decode step of a layer: dqk_append of the
 * step's new K/V rows, then dqk_decode.  Passage: the decode step whose
 * throughput "Throughput on SGLang" reports (cache write + pruned attention).
 *  Arguments: those of dqk_append (k, v, kv_dtype, new_lens, seq_lens_before,
 *  max_new) and of dqk_decode (the rest), same layouts and ownership;
 *  seq_lens must already count the new rows.  All arguments of both parts are
 *  checked before anything is launched.
 *  Result: the same bytes as dqk_append followed by dqk_decode on `stream`.
 *  With max_new <= 4 the append runs inside the decode kernel: its rows are
 *  transformed and packed by the CTAs' prologues next to the query work, and
 *  every page at or past the first page an append touches is read only
 *  after the grid barrier that follows them; longer appends run as their
 *  own kernel first. */
dqk_status dqk_decode_step(const dqk_layer_desc *layer, const void *k, const void *v,
                           dqk_dtype kv_dtype, const int *new_lens, const int *seq_lens_before,
                           int max_new, const void *q, dqk_dtype q_dtype, int batch,
                           const int *seq_lens, const int *page_table, int max_pages,
                           int sparsity_pct, float *out, int16_t *sel_out, void *workspace,
                           size_t workspace_bytes, dqk_stream_t stream);

/* Context-parallel decode (one sequence's pages spread over several GPUs):
 * each rank decodes the pages it holds with dqk_decode_partial, the ranks
 * exchange their records (an all-gather over NCCL), and dqk_merge_partials
 * forms the output.  The pages say nothing about splitting the context or
 * merging partial softmax results; this is flash decoding's log-sum-exp
 * merge carried across ranks, exact up to fp32 rounding.
 *
 * dqk_decode_partial -- dqk_decode over the cached tokens this caller holds
 * (its own pool, page table and token counts seq_lens), writing instead of
 * `out` one record per (sequence, query head): part [batch][Hq][2 + d] fp32 =
 * (m, l, o[d]) with m the running max of the scores in log2 units (scores
 * scaled by log2(e)/sqrt(d)), l = sum of 2^(s - m), o = sum of 2^(s - m) v^.
 * A sequence with no tokens here gives (-inf, 0, 0...).  Same arguments as
 * dqk_decode otherwise; all ranks must use the same q and sparsity_pct. */
dqk_status dqk_decode_partial(const dqk_layer_desc *layer, const void *q, dqk_dtype q_dtype,
                              int batch, const int *seq_lens, const int *page_table,
                              int max_pages, int sparsity_pct, float *part, int16_t *sel_out,
                              void *workspace, size_t workspace_bytes, dqk_stream_t stream);

/* out[b][h] = sum_r 2^(m_r - M) o_r / sum_r 2^(m_r - M) l_r over the n_parts
 * records parts [n_parts][batch][Hq][2 + d] (device, fp32), M = max_r m_r,
 * records taken in index order (the same result on every rank); 0 where no
 * range held tokens.  out (device) fp32 [batch][Hq][d]. */
dqk_status dqk_merge_partials(const float *parts, int n_parts, int batch, int num_q_heads,
                              int head_dim, float *out, dqk_stream_t stream);

/* dqk_test_decode_stall -- TEST ONLY: dqk_decode with a fault injected on
 * the host's request, to exercise the bounded waits.  The producer warp of
 * CTA 0 never arms its second ring stage and every ring wait gives up after
 * 1 ms instead of 1 s: the consumers of CTA 0 stop waiting, the producer
 * drains the copies it issued, every CTA still takes part in both grid
 * barriers, and dqk_last_device_error() then returns DQK_ERR_TIMEOUT.  The
 * outputs are undefined; nothing stays in flight and the next call is
 * unaffected.  Arguments as dqk_decode.  The pages have no counterpart. */
dqk_status dqk_test_decode_stall(const dqk_layer_desc *layer, const void *q, dqk_dtype q_dtype,
                                 int batch, const int *seq_lens, const int *page_table,
                                 int max_pages, int sparsity_pct, float *out, int16_t *sel_out,
                                 void *workspace, size_t workspace_bytes, dqk_stream_t stream);

/* Largest workspace dqk_decode_noalloc can serve: 8 MiB of static device
 * memory per device that loads the library. */
#define DQK_NOALLOC_WORKSPACE_BYTES (8u << 20)

/* dqk_decode_noalloc -- dqk_decode without a caller-provided workspace.
 * The paper has no counterpart: this exists for callers that cannot allocate
 * device memory at decode time -- for example a plugin inside a host engine
 * whose op interface offers no scratch buffer, or a serving loop that forbids
 * allocation once it is warmed up (a cudaMalloc there can stall on the driver
 * or fail when the memory pool is full).
 *  Arguments and results: as dqk_decode, minus workspace/workspace_bytes.
 *  Scratch: a fixed DQK_NOALLOC_WORKSPACE_BYTES array in the library's static
 *  device memory, held by every device that loads the library until the
 *  process exits.  A request needing more than that (see
 *  dqk_decode_workspace_size) returns DQK_ERR_WORKSPACE_TOO_SMALL with nothing
 *  launched.  The call allocates nothing.
 *  Set-up: the first call on a device (with that device current) looks up the
 *  array's device address once; make that first call before any stream
 *  capture.
 *  Sharing: every call on a device uses the same array.  Calls whose work
 *  overlaps on the GPU (different streams, no ordering between them) race on
 *  it; order them on one stream or with events.  The decode needs no zeroed
 *  scratch: each call writes what it reads. */
dqk_status dqk_decode_noalloc(const dqk_layer_desc *layer, const void *q, dqk_dtype q_dtype,
                              int batch, const int *seq_lens, const int *page_table,
                              int max_pages, int sparsity_pct, float *out, int16_t *sel_out,
                              dqk_stream_t stream);

/* ---------------------------------------------------------------------------
 * The BF16 comparison decode: plain attention over a paged BF16 K/V cache, no
 * transform, no quantization, no channel pruning -- the baseline the decode
 * speedup of "Throughput on SGLang" (3.75x over BF16) is quoted against.  It
 * uses the same dqk_layer_desc (t_k, t_q, group_size and v_ch0_protect are
 * ignored; pool holds BF16 blocks) and the same page tables.
 *
 * Block of (page, kv head), 64*d bytes (8192 at d = 128): K [16][d] then
 * V [16][d] BF16, token-major; the 16-byte chunk x (channels 8x..8x+7) of
 * token t is stored at chunk position x ^ (t % 8) of its row.
 * ------------------------------------------------------------------------- */
size_t dqk_bf16_block_bytes(const dqk_layer_desc *layer);

/* Copy new K/V rows into the BF16 cache; arguments as dqk_append (k and v
 * 16-byte aligned; fp32 rows are rounded to BF16, RNE). */
dqk_status dqk_bf16_append(const dqk_layer_desc *layer, const void *k, const void *v, dqk_dtype dtype,
                           int batch, const int *new_lens, const int *seq_lens_before, int max_new,
                           const int *page_table, int max_pages, dqk_stream_t stream);

/* Workspace of dqk_bf16_decode (0 = unsupported). */
size_t dqk_bf16_decode_workspace_size(const dqk_layer_desc *layer, int batch, int max_pages);

/* out = softmax(q.k / sqrt(d)) . v over the first seq_lens[b] cached tokens,
 * every channel kept; arguments as dqk_decode (no sparsity, no sel_out).
 * Query pieces and softmax weights are carried as BF16 hi + lo pairs
 * (about 16 significant bits), accumulation in fp32. */
dqk_status dqk_bf16_decode(const dqk_layer_desc *layer, const void *q, dqk_dtype q_dtype, int batch,
                           const int *seq_lens, const int *page_table, int max_pages, float *out,
                           void *workspace, size_t workspace_bytes, dqk_stream_t stream);

/* Synchronizes `stream`, then reads and clears the current device's error
 * word: DQK_OK, DQK_ERR_DEVICE_BOUNDS or DQK_ERR_TIMEOUT (DQK_ERR_CUDA if the
 * stream itself reports an error).  All calls on a device share the word. */
dqk_status dqk_last_device_error(dqk_stream_t stream);

/* Static, human-readable name of a status. */
const char *dqk_status_string(dqk_status status);

#ifdef __cplusplus
}
#endif
#endif /* DUALQK_H */
