"""Seeded synthetic inputs for the Dual-QK decode path.

This module is the only code that both the CUDA path (tests, bench) and the
CPU oracle draw from.  It holds none of the method's arithmetic: no key or
query transform is applied here, nothing is quantized, selected or attended.
It only draws the raw tensors a serving stack would hand to the library:

* K/V rows as a BF16 (or fp32) model writes them, with RoPE already applied
  (the pages put RoPE before the key transform; rotating is the caller's job),
* the paired transforms T_K and T_Q = T_K^{-T} (synthetic "calibration"),
* decode queries, context lengths and page tables.

Every tensor is a pure function of (workload seed, tensor kind, indices), so
any slice can be regenerated on its own: K/V are drawn in 1024-token chunks
from ``numpy.random.default_rng([seed, kind, b, chunk])`` (PCG64).

Workload recipe (the pages print no inputs; shapes follow the Llama-3-8B and
Qwen3-8B attention layers the Dual-QK page lists among its references):

* ``tiny``     -- 1 kv head, head_dim 64, 1024 tokens, fp32 K/V ~ N(0,1) with
  key channels 3 and 17 scaled x20, T_K = I + 0.1 N(0,1) (cond < 10),
  4 decode queries sharing one page set, 40 % sparsity, no RoPE.
* ``llama``    -- batch 8, 32/8 heads, head_dim 128, 32K tokens, BF16 K/V
  ~ N(0,1), 4 random key outlier channels per kv head x15, RoPE theta 5e5,
  T_K = Cov^{-1/4} of a random SPD covariance, sequential pages.
* ``long``     -- the llama layer at batch 4 and 128K tokens, pages in a seeded
  random order.
* ``qwen``     -- batch 16, 32/8 heads, lengths uniform in [4096, 65536],
  Student-t(3) keys, N(0,1) values, 64 tokens appended before decode,
  RoPE theta 1e6, random page order.
* ``sweep``    -- the ``long`` shape with sparsity, batch and context varied.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

PAGE = 16          # tokens per page
CHUNK = 1024       # tokens per independently seeded K/V draw

# stream ids (second word of every seed sequence)
_S_KV, _S_Q, _S_T, _S_OUTL, _S_LEN, _S_PERM = 11, 12, 13, 14, 15, 16
_S_QBASIS, _S_CAL = 17, 18


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    hq: int
    hkv: int
    d: int
    ctx: int | None              # None: ragged lengths in [ctx_lo, ctx_hi]
    seed: int
    kv_dtype: str = "bf16"       # "bf16" or "f32"
    k_dist: str = "normal"       # "normal" or "t3"
    outliers: str = "random4"    # "fixed_3_17", "random4" or "none"
    transform: str = "whiten"    # "whiten" (Cov^-1/4), "noise" (I + 0.1 N) or "calibrated" (built by the
                                 # caller from calibration_rows; see bit_kv_cache_dqk_b200.calibrate)
    q_dist: str = "normal"       # "normal" or "lowrank" (queries near a rank-8 subspace per kv head)
    rope_theta: float | None = 5e5
    pct: int = 40
    page_order: str = "random"   # "sequential", "random" or "shared"
    append_new: int = 0          # tokens appended just before decode
    ctx_lo: int = 4096
    ctx_hi: int = 65536
    v_ch0_protect: int = 0
    group_size: int = 32         # channels per (scale, min) group: 32, or head_dim (one group per token)
    len_multiple: int = 1        # ragged lengths rounded up to a multiple of this (16: only full pages)

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": Workload("tiny", batch=4, hq=1, hkv=1, d=64, ctx=1024, seed=1,
                     kv_dtype="f32", outliers="fixed_3_17", transform="noise",
                     rope_theta=None, page_order="shared"),
    "llama": Workload("llama", batch=8, hq=32, hkv=8, d=128, ctx=32768, seed=2,
                      page_order="sequential"),
    "long": Workload("long", batch=4, hq=32, hkv=8, d=128, ctx=131072, seed=3),
    "qwen": Workload("qwen", batch=16, hq=32, hkv=8, d=128, ctx=None, seed=4,
                     k_dist="t3", outliers="none", rope_theta=1e6, append_new=64),
    "sweep": Workload("sweep", batch=16, hq=32, hkv=8, d=128, ctx=131072, seed=5),
    # the 128K layer with one (scale, min) group per token (74 B per token and kv head)
    "long128": Workload("long128", batch=4, hq=32, hkv=8, d=128, ctx=131072, seed=3, group_size=128),
    # the llama layer with structured queries and calibrated transforms (next-step row f1)
    "llama_cal": Workload("llama_cal", batch=8, hq=32, hkv=8, d=128, ctx=32768, seed=6,
                          transform="calibrated", q_dist="lowrank", page_order="random"),
}


# ----------------------------------------------------------------------------
# lengths and page tables
# ----------------------------------------------------------------------------
def lengths(w: Workload) -> np.ndarray:
    """Context length of every sequence at decode time (appended rows included)."""
    if w.ctx is not None:
        return np.full(w.batch, w.ctx, dtype=np.int32)
    rng = np.random.default_rng([w.seed, _S_LEN])
    lens = rng.integers(w.ctx_lo, w.ctx_hi + 1, size=w.batch)
    m = w.len_multiple
    return (((lens + m - 1) // m) * m).astype(np.int32)


def page_table(w: Workload, lens: np.ndarray):
    """Logical->physical page map [batch][max_pages] (int32) and the pool size.

    ``shared``: every row maps to the same pages (several queries over one
    sequence).  ``sequential``: sequence b owns a contiguous run.  ``random``:
    a seeded permutation of the whole pool is dealt out in (b, page) order.
    Unused entries are -1.
    """
    npages = (lens.astype(np.int64) + PAGE - 1) // PAGE
    max_pages = int(npages.max()) if len(npages) else 0
    table = np.full((w.batch, max(max_pages, 1)), -1, dtype=np.int32)
    if w.page_order == "shared":
        n = int(npages[0])
        for b in range(w.batch):
            table[b, :n] = np.arange(n)
        return table, n
    total = int(npages.sum())
    if w.page_order == "sequential":
        phys = np.arange(total, dtype=np.int64)
    else:
        phys = np.random.default_rng([w.seed, _S_PERM]).permutation(total)
    off = 0
    for b in range(w.batch):
        n = int(npages[b])
        table[b, :n] = phys[off:off + n]
        off += n
    return table, total


# ----------------------------------------------------------------------------
# transforms (synthetic calibration)
# ----------------------------------------------------------------------------
def _whitening_pair(rng, d):
    a = rng.standard_normal((d, d))
    qm, r = np.linalg.qr(a)
    qm = qm * np.sign(np.diag(r))[None, :]
    lam = 10.0 ** rng.uniform(-1.0, 1.0, size=d)
    t_k = (qm * lam ** -0.25) @ qm.T
    t_q = (qm * lam ** 0.25) @ qm.T
    return t_k, t_q


def _noise_pair(seed, d):
    s = seed
    while True:
        rng = np.random.default_rng([s, _S_T])
        t_k = np.eye(d) + 0.1 * rng.standard_normal((d, d))
        if np.linalg.cond(t_k) < 10.0:
            return t_k, np.linalg.inv(t_k).T, s
        s += 1


def transforms(w: Workload):
    """(t_k32, t_q32, t_k64, t_q64), each [hkv][d][d] row-major.

    ``whiten``: Cov = Q diag(lam) Q^T with Q from the sign-fixed QR of a
    seeded Gaussian matrix and lam = 10^U(-1,1); T_K = Cov^{-1/4} and
    T_Q = Cov^{1/4} (= T_K^{-T}, T_K being symmetric), built in fp64.
    ``noise``: T_K = I + 0.1 N(0,1), redrawn with seed+1 until cond < 10,
    T_Q = inv(T_K)^T.
    """
    if w.transform == "calibrated":
        raise ValueError("calibrated transforms are built from calibration_rows by the calibrate module")
    t_k = np.empty((w.hkv, w.d, w.d))
    t_q = np.empty((w.hkv, w.d, w.d))
    for j in range(w.hkv):
        if w.transform == "noise":
            t_k[j], t_q[j], _ = _noise_pair(w.seed + 1000 * j, w.d)
        elif w.transform == "identity":
            t_k[j] = np.eye(w.d)
            t_q[j] = np.eye(w.d)
        else:
            t_k[j], t_q[j] = _whitening_pair(np.random.default_rng([w.seed, _S_T, j]), w.d)
    return (t_k.astype(np.float32), t_q.astype(np.float32), t_k, t_q)


# ----------------------------------------------------------------------------
# K/V rows and queries
# ----------------------------------------------------------------------------
def _outlier_gain(w: Workload) -> np.ndarray:
    """Per (kv head, channel) gain applied to raw keys."""
    gain = np.ones((w.hkv, w.d), dtype=np.float32)
    if w.outliers == "fixed_3_17":
        gain[:, [3, 17]] = 20.0
    elif w.outliers == "random4":
        rng = np.random.default_rng([w.seed, _S_OUTL])
        for j in range(w.hkv):
            gain[j, rng.choice(w.d, size=4, replace=False)] = 15.0
    return gain


def _rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE: pairs (i, i+d/2), inv_freq_i = theta^(-2i/d).

    x: [..., n, heads, d] float32 with positions ``pos`` [n]; computed in fp64.
    """
    d = x.shape[-1]
    half = d // 2
    inv = theta ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = pos.astype(np.float64)[:, None] * inv[None, :]            # [n, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1 = x[..., :half].astype(np.float64)
    x2 = x[..., half:].astype(np.float64)
    out = np.empty(x.shape, dtype=np.float64)
    out[..., :half] = x1 * c - x2 * s
    out[..., half:] = x2 * c + x1 * s
    return out.astype(np.float32)


def _to_model_dtype(x: np.ndarray, kv_dtype: str) -> np.ndarray:
    """Round fp32 values to what the model hands over (BF16 RNE), kept as fp32."""
    if kv_dtype == "f32":
        return x
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)
    return t.to(torch.float32).numpy()


def _kv_chunk(w: Workload, b: int, c: int, gain: np.ndarray):
    rng = np.random.default_rng([w.seed, _S_KV, b, c])
    shape = (CHUNK, w.hkv, w.d)
    if w.k_dist == "t3":
        k = rng.standard_t(3, size=shape).astype(np.float32)
    else:
        k = np.empty(shape, dtype=np.float32)
        rng.standard_normal(out=k, dtype=np.float32)
    v = np.empty(shape, dtype=np.float32)
    rng.standard_normal(out=v, dtype=np.float32)
    k *= gain[None]
    if w.rope_theta is not None:
        k = _rope(k, np.arange(c * CHUNK, (c + 1) * CHUNK), w.rope_theta)
    return _to_model_dtype(k, w.kv_dtype), _to_model_dtype(v, w.kv_dtype)


def kv_rows(w: Workload, b: int, t0: int, t1: int, threads: int = 8):
    """Keys and values of sequence ``b``, positions [t0, t1): two fp32 arrays
    [t1-t0][hkv][d] holding model-dtype values (RoPE already on the keys)."""
    n = t1 - t0
    k = np.empty((n, w.hkv, w.d), dtype=np.float32)
    v = np.empty((n, w.hkv, w.d), dtype=np.float32)
    if n <= 0:
        return k, v
    gain = _outlier_gain(w)
    chunks = range(t0 // CHUNK, (t1 - 1) // CHUNK + 1)

    def fill(c):
        kc, vc = _kv_chunk(w, b, c, gain)
        lo = max(t0, c * CHUNK)
        hi = min(t1, (c + 1) * CHUNK)
        k[lo - t0:hi - t0] = kc[lo - c * CHUNK:hi - c * CHUNK]
        v[lo - t0:hi - t0] = vc[lo - c * CHUNK:hi - c * CHUNK]

    if threads > 1 and len(chunks) > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, chunks))
    else:
        for c in chunks:
            fill(c)
    return k, v


def kv_rows_device(w: Workload, seqs, t0: int, t1: int, device):
    """Large-sweep stand-in for ``kv_rows``: keys and values of sequences
    ``seqs``, positions [t0, t1), drawn on the device with torch's Philox
    generator (seeded by (seed, chunk)), same distributions as ``kv_rows``
    (N(0,1) or Student-t(3) keys times the outlier gains, N(0,1) values,
    rotate-half RoPE, model dtype).  Returns two tensors [len(seqs)*(t1-t0)]
    [hkv][d], sequence-major.  Not bit-identical to ``kv_rows``; used where the
    CPU draw would take minutes and no oracle comparison is made."""
    import torch
    n = t1 - t0
    g = torch.Generator(device=device)
    g.manual_seed(int(w.seed) * 1000003 + int(t0))
    shape = (len(seqs), n, w.hkv, w.d)
    if w.k_dist == "t3":
        z = torch.randn(shape, generator=g, device=device)
        chi = torch.randn((3,) + shape, generator=g, device=device).pow(2).sum(0)
        k = z / torch.sqrt(chi / 3.0)
    else:
        k = torch.randn(shape, generator=g, device=device)
    v = torch.randn(shape, generator=g, device=device)
    k = k * torch.from_numpy(_outlier_gain(w)).to(device)[None, None]
    if w.rope_theta is not None:
        half = w.d // 2
        inv = torch.tensor(w.rope_theta ** (-np.arange(half, dtype=np.float64) * 2.0 / w.d), device=device)
        ang = torch.arange(t0, t1, device=device, dtype=torch.float64)[:, None] * inv[None, :]
        c = torch.cos(ang).float()[None, :, None, :]
        sn = torch.sin(ang).float()[None, :, None, :]
        k1, k2 = k[..., :half], k[..., half:]
        k = torch.cat([k1 * c - k2 * sn, k2 * c + k1 * sn], dim=-1)
    dt = torch.bfloat16 if w.kv_dtype == "bf16" else torch.float32
    return k.to(dt).reshape(-1, w.hkv, w.d).contiguous(), v.to(dt).reshape(-1, w.hkv, w.d).contiguous()


_QRANK = 8
_QSCALES = np.array([4.0, 3.0, 2.5, 2.0, 1.6, 1.3, 1.0, 0.8])


def _query_basis(w: Workload) -> np.ndarray:
    """Per kv head, an orthonormal d x 8 basis the ``lowrank`` queries live near."""
    rng = np.random.default_rng([w.seed, _S_QBASIS])
    out = np.empty((w.hkv, w.d, _QRANK))
    for j in range(w.hkv):
        qm, _ = np.linalg.qr(rng.standard_normal((w.d, _QRANK)))
        out[j] = qm
    return out


def _raw_queries(w: Workload, rng, rows: int) -> np.ndarray:
    """[rows][hq][d] pre-RoPE queries of the workload's distribution."""
    if w.q_dist == "lowrank":
        basis = _query_basis(w)
        z = rng.standard_normal((rows, w.hq, _QRANK)) * _QSCALES[None, None, :]
        q = np.einsum("hdr,nhr->nhd", basis[np.arange(w.hq) // w.group], z)   # head h near its kv head's subspace
        q += 0.25 * rng.standard_normal((rows, w.hq, w.d))
        return q.astype(np.float32)
    return rng.standard_normal((rows, w.hq, w.d)).astype(np.float32)


def calibration_rows(w: Workload, n_keys: int = 4096, n_queries: int = 1024):
    """Calibration activations: keys [n_keys][hkv][d] and queries
    [n_queries][hq][d] of the workload's distributions, RoPE'd at seeded random
    positions within the context, in model dtype (fp32 arrays).  Drawn from
    their own streams, disjoint from the decoded rows."""
    rng = np.random.default_rng([w.seed, _S_CAL])
    ctx = w.ctx if w.ctx is not None else w.ctx_hi
    gain = _outlier_gain(w)
    if w.k_dist == "t3":
        k = rng.standard_t(3, size=(n_keys, w.hkv, w.d)).astype(np.float32)
    else:
        k = rng.standard_normal((n_keys, w.hkv, w.d)).astype(np.float32)
    k *= gain[None]
    q = _raw_queries(w, rng, n_queries)
    if w.rope_theta is not None:
        pk = rng.integers(0, ctx, size=n_keys)
        pq = rng.integers(0, ctx, size=n_queries)
        k = np.concatenate([_rope(k[i:i + 1], pk[i:i + 1], w.rope_theta) for i in range(n_keys)])
        q = np.concatenate([_rope(q[i:i + 1], pq[i:i + 1], w.rope_theta) for i in range(n_queries)])
    return _to_model_dtype(k, w.kv_dtype), _to_model_dtype(q, w.kv_dtype)


def queries(w: Workload, lens: np.ndarray, step: int = 0) -> np.ndarray:
    """Decode queries [batch][hq][d] (fp32 holding model-dtype values), RoPE'd
    at position L_b - 1.  ``step`` selects an independent draw."""
    rng = np.random.default_rng([w.seed, _S_Q, step])
    q = _raw_queries(w, rng, w.batch)
    if w.rope_theta is not None:
        for b in range(w.batch):
            q[b] = _rope(q[b][None], np.array([int(lens[b]) - 1]), w.rope_theta)[0]
    return _to_model_dtype(q, w.kv_dtype)


def describe(w: Workload) -> dict:
    lens = lengths(w)
    return {"workload": w.name, "batch": w.batch, "q_heads": w.hq, "kv_heads": w.hkv,
            "head_dim": w.d, "context": int(lens.max()) if w.ctx is None else w.ctx,
            "ragged": w.ctx is None, "sparsity_pct": w.pct, "page_tokens": PAGE,
            "page_order": w.page_order, "kv_dtype": w.kv_dtype, "seed": w.seed,
            "tokens_per_step": int(lens.sum())}


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["Workload", "CONFIGS", "PAGE", "lengths", "page_table", "transforms",
           "kv_rows", "kv_rows_device", "queries", "calibration_rows", "describe", "ceil_div"]
