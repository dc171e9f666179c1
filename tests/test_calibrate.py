"""The calibrated transform pair (next-step row f1), CPU only.

The oracle's construction (cyclic Jacobi in plain C) is pinned by what the
definition fixes -- T_Q = T_K^-T, the key spectrum becomes lambda^(1-alpha),
the query second moment becomes diagonal and sorted, alpha = 0 gives an
orthogonal PCA basis, a hand-built diagonal case -- and the package's
construction (LAPACK through numpy) must agree with it."""
import numpy as np
import pytest

from bit_kv_cache_dqk_b200 import calibrate as Cb
from bit_kv_cache_dqk_b200 import inputs as I


def _data(seed, d, n=600, m=400):
    rng = np.random.default_rng(seed)
    scales = np.linspace(0.5, 6.0, d)
    k = rng.standard_normal((n, d)) * scales
    q = rng.standard_normal((m, d)) @ rng.standard_normal((d, d))
    return k, q


@pytest.mark.parametrize("d,alpha", [(8, 0.5), (16, 0.5), (16, 1.0), (32, 0.25)])
def test_oracle_pair_definition(oracle_mod, d, alpha):
    k, q = _data(d, d)
    tk, tq = oracle_mod.calibrate(k, q, alpha)
    assert np.abs(tq @ tk.T - np.eye(d)).max() < 1e-11              # T_Q = T_K^-T
    ck = k.T @ k / len(k)
    ck += np.eye(d) * (1e-6 * np.trace(ck) / d)
    lam = np.linalg.eigvalsh(ck)
    got = np.linalg.eigvalsh(tk @ ck @ tk.T)
    assert np.allclose(np.sort(got), np.sort(lam ** (1.0 - alpha)), rtol=1e-9)
    cq = tq @ (q.T @ q / len(q)) @ tq.T
    off = cq - np.diag(np.diag(cq))
    assert np.abs(off).max() < 1e-9 * np.abs(cq).max()              # decorrelated
    assert np.all(np.diff(np.diag(cq)) <= 1e-9 * cq[0, 0])           # energy sorted
    kk, qq = k[:5], q[:5]
    assert np.allclose((qq @ tq.T) @ (kk @ tk.T).T, qq @ kk.T, rtol=1e-10, atol=1e-10)


def test_oracle_alpha0_is_query_pca(oracle_mod):
    k, q = _data(3, 12)
    tk, tq = oracle_mod.calibrate(k, q, 0.0)
    assert np.abs(tk - tq).max() < 1e-12
    assert np.abs(tk @ tk.T - np.eye(12)).max() < 1e-12
    mu, u = np.linalg.eigh(q.T @ q / len(q))
    assert np.allclose(np.abs(tq[0]), np.abs(u[:, -1]), atol=1e-9)   # row 0 = dominant query direction


def test_oracle_hand_built_diagonal_case(oracle_mod):
    """C_K = diag(16, 1, 81, 1) and queries along axes 3 (strong), 1, 0, 2:
    P = diag(2, 1, 3, 1) (alpha 1/2), the basis is a signed permutation, so T_K
    and T_Q are permutation matrices times diag(1/2, 1, 1/3, 1) and diag(2, 1, 3, 1)."""
    d = 4
    k = np.zeros((4, d))
    k[0, 0], k[1, 1], k[2, 2], k[3, 3] = 8.0, 2.0, 18.0, 2.0       # K^T K / 4 = diag(16, 1, 81, 1)
    q = np.zeros((4, d))
    q[0, 3], q[1, 1], q[2, 0], q[3, 2] = 10.0, 5.0, 1.0, 0.1         # energies after P: 100, 25, 4, 0.09
    tk, tq = oracle_mod.calibrate(k, q, 0.5)
    eps = 1e-6 * (16 + 1 + 81 + 1) / d     # 1e-6 * trace(C_K) / d
    p = np.sqrt(np.sqrt(np.array([16.0, 1.0, 81.0, 1.0]) + eps))
    order = [3, 1, 0, 2]
    exp_q = np.zeros((d, d))
    exp_k = np.zeros((d, d))
    for c, a in enumerate(order):
        exp_q[c, a] = p[a]
        exp_k[c, a] = 1.0 / p[a]
    assert np.abs(tq - exp_q).max() < 1e-12 and np.abs(tk - exp_k).max() < 1e-12


@pytest.mark.parametrize("d", [16, 64])
def test_package_matches_oracle(oracle_mod, d):
    k, q = _data(7 + d, d, n=900, m=700)
    tk_o, tq_o = oracle_mod.calibrate(k, q, 0.5)
    tk_p, tq_p = Cb.calibrate_head(k, q, 0.5)
    assert np.abs(tk_o - tk_p).max() < 1e-8 * np.abs(tk_o).max()
    assert np.abs(tq_o - tq_p).max() < 1e-8 * np.abs(tq_o).max()


def test_calibration_concentrates_query_energy():
    """With queries near a low-rank subspace, the calibrated pair keeps more of
    the query energy under 40 % pruning than the uncalibrated whitening pair."""
    w = I.CONFIGS["llama_cal"].with_(batch=4, hkv=2, hq=8)
    k, q = I.calibration_rows(w, n_keys=2048, n_queries=512)
    _, _, tk, tq = Cb.calibrate_layer(k, q)
    qd = I.queries(w, np.full(w.batch, 4096))
    keep = w.d - (40 * w.d) // 100
    cal = Cb.energy_kept(tq, qd, keep, w.group)
    _, _, _, tqw = I.transforms(w.with_(transform="whiten"))
    base = Cb.energy_kept(tqw, qd, keep, w.group)
    assert cal > 0.98 and cal > base + 0.01
