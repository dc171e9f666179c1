"""ctypes front end of the fp64 CPU oracle (``liboracle.so``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / reference leg of ``bench.py``; never by the
product package.  See ``dualqk_oracle.c`` for what each function computes
and which page passages it follows.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dualqk_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
GROUP = 32


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared",
               "-ffp-contract=off", "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        P = C.c_void_p
        _lib.oracle_f64_to_f16.restype = C.c_uint16
        _lib.oracle_f64_to_f16.argtypes = [C.c_double]
        _lib.oracle_f16_to_f64.restype = C.c_double
        _lib.oracle_f16_to_f64.argtypes = [C.c_uint16]
        _lib.oracle_f32_to_bf16.restype = C.c_uint16
        _lib.oracle_f32_to_bf16.argtypes = [C.c_float]
        _lib.oracle_bf16_to_f64.restype = C.c_double
        _lib.oracle_bf16_to_f64.argtypes = [C.c_uint16]
        _lib.oracle_transform_f32.argtypes = [C.c_int, P, P, P]
        _lib.oracle_transform_f64.argtypes = [C.c_int, P, P, P]
        _lib.oracle_quantize_vec.argtypes = [C.c_int, P, C.c_int, P, P, P, P]
        _lib.oracle_append.restype = C.c_int
        _lib.oracle_append.argtypes = [C.c_int, C.c_int, C.c_int, P, P, P, C.c_longlong,
                                       P, P, P, P, P, P, P, P]
        _lib.oracle_n_keep.restype = C.c_int
        _lib.oracle_n_keep.argtypes = [C.c_int, C.c_int]
        _lib.oracle_select.argtypes = [C.c_int, P, C.c_int, P]
        _lib.oracle_qprep.argtypes = [C.c_int, P, P, C.c_int, P, P]
        _lib.oracle_decode_seq.restype = C.c_int
        _lib.oracle_decode_seq.argtypes = [C.c_int] * 6 + [P] * 10 + [P, P, P, C.c_int]
        _lib.oracle_decode_dense.restype = C.c_int
        _lib.oracle_decode_dense.argtypes = [C.c_int] * 5 + [P] * 7
        _lib.oracle_quantize_vec_g.argtypes = [C.c_int, C.c_int, P, C.c_int, P, P, P, P]
        _lib.oracle_append_g.restype = C.c_int
        _lib.oracle_append_g.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, P, P, P, C.c_longlong,
                                         P, P, P, P, P, P, P, P]
        _lib.oracle_decode_seq_g.restype = C.c_int
        _lib.oracle_decode_seq_g.argtypes = [C.c_int] * 7 + [P] * 10 + [P, P, P, C.c_int]
        _lib.oracle_calibrate.restype = C.c_int
        _lib.oracle_calibrate.argtypes = [C.c_int, C.c_longlong, C.c_longlong, C.c_double, P, P, P, P]
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


# ---------------------------------------------------------------- conversions
def f64_to_f16_bits(x: float) -> int:
    return int(lib().oracle_f64_to_f16(float(x)))


def f16_bits_to_f64(h: int) -> float:
    return float(lib().oracle_f16_to_f64(int(h)))


def f32_to_bf16_bits(x: float) -> int:
    return int(lib().oracle_f32_to_bf16(float(np.float32(x))))


def bf16_bits_to_f64(b: int) -> float:
    return float(lib().oracle_bf16_to_f64(int(b)))


# ---------------------------------------------------------------- method steps
def transform_f32(t: np.ndarray, x: np.ndarray) -> np.ndarray:
    t, x = _f32(t), _f32(x)
    d = x.shape[-1]
    y = np.empty(d, dtype=np.float32)
    lib().oracle_transform_f32(d, _p(t), _p(x), _p(y))
    return y


def quantize_vec(x: np.ndarray, protect_ch0: bool, gs: int = GROUP):
    """One token vector: codes, fp16 scale/min per group of gs channels, BF16 ch0."""
    x = _f32(x)
    d = x.shape[0]
    codes = np.empty(d, dtype=np.uint8)
    scale = np.empty(d // gs, dtype=np.uint16)
    mn = np.empty(d // gs, dtype=np.uint16)
    ch0 = np.zeros(1, dtype=np.uint16)
    lib().oracle_quantize_vec_g(d, gs, _p(x), int(protect_ch0), _p(codes), _p(scale), _p(mn), _p(ch0))
    return codes, scale, mn, int(ch0[0])


def n_keep(d: int, pct: int) -> int:
    return int(lib().oracle_n_keep(d, pct))


def select(absq: np.ndarray, keep: int) -> np.ndarray:
    a = _f64(absq)
    sel = np.empty(keep, dtype=np.int16)
    lib().oracle_select(a.shape[0], _p(a), keep, _p(sel))
    return sel


def qprep(t_q_head: np.ndarray, q: np.ndarray, pct: int):
    """q' (fp32) and the selected channels (ascending) of one query head."""
    t, q = _f32(t_q_head), _f32(q)
    d = q.shape[0]
    qp = np.empty(d, dtype=np.float32)
    sel = np.empty(n_keep(d, pct), dtype=np.int16)
    lib().oracle_qprep(d, _p(t), _p(q), pct, _p(qp), _p(sel))
    return qp, sel


class Cache(dict):
    """Plain quantized rows of one sequence: kcodes/vcodes [n][hkv][d] uint8,
    kscale/kmin/vscale/vmin [n][hkv][d/32] fp16 bits, kch0/vch0 [n][hkv]."""


def append(t_k: np.ndarray, k: np.ndarray, v: np.ndarray, v_ch0: bool = False, gs: int = GROUP) -> Cache:
    """Transform and quantize rows k, v [n][hkv][d] (fp32 values); scale groups
    of gs channels (32, or d for one group per token)."""
    t_k, k, v = _f32(t_k), _f32(k), _f32(v)
    n, hkv, d = k.shape
    ng = d // gs
    c = Cache(
        kcodes=np.empty((n, hkv, d), np.uint8), kscale=np.empty((n, hkv, ng), np.uint16),
        kmin=np.empty((n, hkv, ng), np.uint16), kch0=np.empty((n, hkv), np.uint16),
        vcodes=np.empty((n, hkv, d), np.uint8), vscale=np.empty((n, hkv, ng), np.uint16),
        vmin=np.empty((n, hkv, ng), np.uint16), vch0=np.empty((n, hkv), np.uint16))
    rc = lib().oracle_append_g(d, gs, hkv, int(v_ch0), _p(t_k), _p(k), _p(v), n,
                               _p(c["kcodes"]), _p(c["kscale"]), _p(c["kmin"]), _p(c["kch0"]),
                               _p(c["vcodes"]), _p(c["vscale"]), _p(c["vmin"]), _p(c["vch0"]))
    if rc:
        raise ValueError(f"oracle_append failed ({rc})")
    return c


def concat(caches) -> Cache:
    return Cache({k: np.concatenate([c[k] for c in caches]) for k in caches[0]})


def decode_seq(cache: Cache, q: np.ndarray, t_q: np.ndarray, hq: int, pct: int,
               v_ch0: bool = False, L: int | None = None, threads: int = 8):
    """Attention of the hq query heads q [hq][d] over the first L rows of one
    sequence's quantized cache.  Returns (out [hq][d] fp64, sel [hq][n_keep],
    qprime [hq][d] fp32)."""
    q, t_q = _f32(q), _f32(t_q)
    n, hkv, d = cache["kcodes"].shape
    L = n if L is None else L
    keep = n_keep(d, pct)
    out = np.empty((hq, d), np.float64)
    sel = np.empty((hq, keep), np.int16)
    qp = np.empty((hq, d), np.float32)
    cc = {k: np.ascontiguousarray(a) for k, a in cache.items()}
    gs = d // cache["kscale"].shape[2]          # scale-group size the cache was built with
    rc = lib().oracle_decode_seq_g(d, gs, hq, hkv, int(v_ch0), pct, L,
                                 _p(cc["kcodes"]), _p(cc["kscale"]), _p(cc["kmin"]), _p(cc["kch0"]),
                                 _p(cc["vcodes"]), _p(cc["vscale"]), _p(cc["vmin"]), _p(cc["vch0"]),
                                 _p(q), _p(t_q), _p(out), _p(sel), _p(qp), threads)
    if rc:
        raise ValueError(f"oracle_decode_seq failed ({rc})")
    return out, sel, qp


LOG2E = 1.4426950408889634


def decode_partial(cache: Cache, q: np.ndarray, t_q: np.ndarray, hq: int, pct: int,
                   v_ch0: bool = False, t0: int = 0, t1: int | None = None) -> np.ndarray:
    """Unnormalized attention record of the rows [t0, t1) of one sequence (the
    split-K combine of the decode path, taken over a row range): for each
    query head, with s_t the pruned score of row t (q'_sel . k^'_sel / sqrt(d))
    written in log2 units u_t = s_t log2(e),
        m = max_t u_t,   l = sum_t 2^(u_t - m),   o = sum_t 2^(u_t - m) v^_t.
    Returns rec [hq][2 + d] fp64 = (m, l, o); (-inf, 0, 0) for an empty range.
    Softmax over the union of ranges is then the merge below."""
    n, hkv, d = cache["kcodes"].shape
    t1 = n if t1 is None else t1
    g = hq // hkv
    rec = np.zeros((hq, 2 + d))
    rec[:, 0] = -np.inf
    if t1 <= t0:
        return rec
    part = Cache({k: a[t0:t1] for k, a in cache.items()})
    kd, vd = dequant(part, v_ch0)
    for h in range(hq):
        j = h // g
        qp, sel = qprep(np.asarray(t_q)[j], np.asarray(q)[h], pct)
        sel = sel.astype(np.int64)
        u = (kd[:, j, sel] @ qp[sel].astype(np.float64)) / np.sqrt(d) * LOG2E
        m = u.max()
        p = np.exp2(u - m)
        rec[h, 0], rec[h, 1] = m, p.sum()
        rec[h, 2:] = p @ vd[:, j, :]
    return rec


def merge_partials(recs: np.ndarray) -> np.ndarray:
    """Output of attention over the union of the ranges of the records recs
    [n][..][2 + d]: sum_r 2^(m_r - M) o_r / sum_r 2^(m_r - M) l_r, M = max_r m_r;
    0 where no range held a row."""
    recs = np.asarray(recs, np.float64)
    m = recs[..., 0]
    top = m.max(axis=0)
    safe = np.where(np.isfinite(top), top, 0.0)
    wgt = np.where(np.isfinite(m), np.exp2(m - safe[None]), 0.0)
    den = (wgt * recs[..., 1]).sum(axis=0)
    num = (wgt[..., None] * recs[..., 2:]).sum(axis=0)
    return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)


def decode_dense(t_k64, t_q64, k, v, q, pct: int, want_scores: bool = False):
    """Quantization-off attention, fp64 throughout.  k, v [L][hkv][d]; q [hq][d]."""
    t_k64, t_q64, k, v, q = map(_f64, (t_k64, t_q64, k, v, q))
    L, hkv, d = k.shape
    hq = q.shape[0]
    out = np.empty((hq, d), np.float64)
    scores = np.empty((hq, L), np.float64) if want_scores else None
    rc = lib().oracle_decode_dense(d, hq, hkv, pct, L, _p(t_k64), _p(t_q64), _p(k), _p(v),
                                   _p(q), _p(out), _p(scores))
    if rc:
        raise ValueError(f"oracle_decode_dense failed ({rc})")
    return (out, scores) if want_scores else out


def dequant(cache: Cache, v_ch0: bool = False):
    """Dequantized (k^', v^) [n][hkv][d] fp64 from the stored fields."""
    n, hkv, d = cache["kcodes"].shape
    f16 = np.vectorize(f16_bits_to_f64, otypes=[np.float64])
    bf = np.vectorize(bf16_bits_to_f64, otypes=[np.float64])
    grp = np.arange(d) // (d // cache["kscale"].shape[2])
    out = []
    for pre, prot in (("k", True), ("v", v_ch0)):
        s = f16(cache[pre + "scale"])[..., grp]
        m = f16(cache[pre + "min"])[..., grp]
        x = m + cache[pre + "codes"].astype(np.float64) * s
        if prot:
            x[..., 0] = bf(cache[pre + "ch0"])
        out.append(x)
    return out[0], out[1]


def calibrate(k: np.ndarray, q: np.ndarray, alpha: float = 0.5):
    """Calibrated transform pair of one kv head from calibration keys k [n][d]
    and queries q [m][d] (fp64 results T_K, T_Q; see oracle_calibrate)."""
    k, q = _f64(k), _f64(q)
    d = k.shape[1]
    t_k = np.empty((d, d), np.float64)
    t_q = np.empty((d, d), np.float64)
    rc = lib().oracle_calibrate(d, k.shape[0], q.shape[0], float(alpha), _p(k), _p(q), _p(t_k), _p(t_q))
    if rc:
        raise ValueError(f"oracle_calibrate failed ({rc})")
    return t_k, t_q
