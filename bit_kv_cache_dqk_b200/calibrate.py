"""Calibrated transform pair (the step before the decode path).

"How does Dual-QK compress KV caches to 2-bit while keeping accuracy at 128K
context?", section "Paired transforms instead of shared rotation": the key
transform combines partial key whitening with a query-aligned basis, guided
by calibrated query and key statistics; it flattens keys for INT2 storage
while the paired query transform concentrates query energy for channel
pruning, and the two preserve query-key dot products.

Construction (offline, fp64, per kv head j, from calibration keys K [n][d]
and the queries of the G query heads of j, Q [m][d], RoPE applied):

    C_K = K^T K / n + eps I                 eps = 1e-6 * trace(K^T K / n) / d
    P   = C_K^(alpha/2)                     partial whitening (alpha = 1/2 by default)
    C_Q = P (Q^T Q / m) P                   query second moment in that frame
    C_Q = U diag(mu) U^T                    mu descending; each column of U signed
                                            so its largest-magnitude entry is > 0
    T_K = U^T P^-1,   T_Q = U^T P           so T_Q = T_K^-T and (T_Q q).(T_K k) = q.k

Channel c of the transformed frame is the c-th strongest query direction, so
channel 0 (kept in BF16 for keys and never pruned) is the dominant one, and
the key spectrum becomes lambda^(1 - alpha).  The library takes the fp32
matrices as T_K and T_Q in dqk_layer_desc.
"""
from __future__ import annotations

import numpy as np


def calibrate_head(k: np.ndarray, q: np.ndarray, alpha: float = 0.5) -> tuple[np.ndarray, np.ndarray]:
    """(T_K, T_Q) in fp64 for one kv head; k [n][d], q [m][d]."""
    k = np.asarray(k, np.float64)
    q = np.asarray(q, np.float64)
    n, d = k.shape
    ck = k.T @ k / n
    ck += np.eye(d) * (1e-6 * np.trace(ck) / d)
    lam, v = np.linalg.eigh(ck)
    p = (v * lam ** (alpha / 2.0)) @ v.T
    p_inv = (v * lam ** (-alpha / 2.0)) @ v.T
    cq = p @ (q.T @ q / q.shape[0]) @ p
    mu, u = np.linalg.eigh((cq + cq.T) / 2.0)
    order = np.argsort(-mu, kind="stable")
    u = u[:, order]
    lead = np.argmax(np.abs(u), axis=0)                 # lowest index among equal magnitudes
    u = u * np.where(u[lead, np.arange(d)] < 0.0, -1.0, 1.0)[None, :]
    return u.T @ p_inv, u.T @ p


def calibrate_layer(k: np.ndarray, q: np.ndarray, alpha: float = 0.5):
    """Transforms of a layer: k [n][hkv][d] calibration keys, q [m][hq][d]
    calibration queries (query head h belongs to kv head h // (hq // hkv)).
    Returns (t_k32, t_q32, t_k64, t_q64), each [hkv][d][d]."""
    n, hkv, d = k.shape
    hq = q.shape[1]
    g = hq // hkv
    t_k = np.empty((hkv, d, d))
    t_q = np.empty((hkv, d, d))
    for j in range(hkv):
        qj = q[:, j * g:(j + 1) * g, :].reshape(-1, d)
        t_k[j], t_q[j] = calibrate_head(k[:, j, :], qj, alpha)
    return t_k.astype(np.float32), t_q.astype(np.float32), t_k, t_q


def energy_kept(t_q: np.ndarray, q: np.ndarray, keep: int, g: int) -> float:
    """Mean fraction of |q'|^2 held by the `keep` largest-|q'| channels (channel
    0 always among them) over the query rows q [m][hq][d] -- how much of the
    score a pruned query retains."""
    m, hq, d = q.shape
    fr = []
    for h in range(hq):
        qp = np.asarray(q[:, h, :], np.float64) @ np.asarray(t_q[h // g], np.float64).T
        e = qp ** 2
        rest = np.sort(e[:, 1:], axis=1)[:, ::-1][:, :keep - 1].sum(axis=1)
        fr.append(((e[:, 0] + rest) / e.sum(axis=1)).mean())
    return float(np.mean(fr))


def layer_transforms(w):
    """(t_k32, t_q32, t_k64, t_q64) of a workload: calibrated from its
    calibration rows when ``w.transform == "calibrated"``, else the synthetic
    pair of ``inputs.transforms``."""
    from . import inputs as I
    if w.transform == "calibrated":
        k, q = I.calibration_rows(w)
        return calibrate_layer(k, q)
    return I.transforms(w)
