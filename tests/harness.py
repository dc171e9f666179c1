"""Test harness: drives libdualqk on a device and computes the oracle's answer
for the same seeded workload.

* ``DeviceRun`` allocates the layer (pool, transforms, tables) with torch and
  calls the C ABI through the ctypes binding.
* ``decode_pool`` reads the packed cache back into plain per-token arrays,
  following the block layout documented in include/dualqk.h (independently of
  the CUDA sources).
* ``oracle_reference`` quantizes the same rows with the CPU oracle and decodes.
"""
from __future__ import annotations

import os

import numpy as np
import torch

from bit_kv_cache_dqk_b200 import dualqk as Q
from bit_kv_cache_dqk_b200 import inputs as I
from oracle import oracle as O

ATOL = 2e-3          # max abs error on fp32 outputs
PARITY_RECORDS = []  # (test, max abs error, max row-relative error) of every output comparison
RTOL_ROW = 1e-2      # relative error per output row (||o - o_ref|| / ||o_ref||)


_TRANSFORMS = {}


def workload_transforms(w: I.Workload):
    """(t_k32, t_q32, t_k64, t_q64) of a workload, the same arrays for the device
    and the oracle.  Calibrated pairs are built by the oracle's own calibration
    from the workload's calibration rows."""
    key = w
    if key not in _TRANSFORMS:
        if w.transform == "calibrated":
            k, q = I.calibration_rows(w)
            g = w.hq // w.hkv
            tk = np.empty((w.hkv, w.d, w.d))
            tq = np.empty((w.hkv, w.d, w.d))
            for j in range(w.hkv):
                tk[j], tq[j] = O.calibrate(k[:, j, :], q[:, j * g:(j + 1) * g, :].reshape(-1, w.d))
            _TRANSFORMS[key] = (tk.astype(np.float32), tq.astype(np.float32), tk, tq)
        else:
            _TRANSFORMS[key] = I.transforms(w)
    return _TRANSFORMS[key]


def torch_dtype(w):
    return torch.bfloat16 if w.kv_dtype == "bf16" else torch.float32


def lib_dtype(w):
    return Q.DQK_BF16 if w.kv_dtype == "bf16" else Q.DQK_F32


class DeviceRun:
    def __init__(self, w: I.Workload, device: str = "cuda:0", lens=None, fill: int = 0xA5):
        self.w = w
        self.dev = torch.device(device)
        self.lens = I.lengths(w) if lens is None else np.asarray(lens, dtype=np.int32)
        self.table, self.num_pages = I.page_table(w, np.maximum(self.lens, 1))
        self.max_pages = self.table.shape[1]
        tk, tq, _, _ = workload_transforms(w)
        self.tk_host, self.tq_host = tk, tq
        self.t_k = torch.from_numpy(tk).to(self.dev)
        self.t_q = torch.from_numpy(tq).to(self.dev)
        probe = Q.layer_desc(w.d, w.hq, w.hkv, 0, 0, 0, 1, v_ch0_protect=w.v_ch0_protect,
                             group_size=w.group_size)
        self.block_bytes = Q.dqk_block_bytes(probe)
        self.pool = torch.full((self.num_pages * w.hkv * self.block_bytes,), fill, dtype=torch.uint8,
                               device=self.dev)
        self.desc = Q.layer_desc(w.d, w.hq, w.hkv, self.t_k, self.t_q, self.pool, self.num_pages,
                                 v_ch0_protect=w.v_ch0_protect, group_size=w.group_size)
        self.table_dev = torch.from_numpy(self.table).to(self.dev)
        self.cached = np.zeros(w.batch, dtype=np.int32)      # tokens appended so far
        self.ws_bytes = Q.dqk_decode_workspace_size(self.desc, w.batch, self.max_pages)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.dev)

    # sequences whose rows are appended (the shared-page workload appends once)
    def _writers(self):
        return [0] if self.w.page_order == "shared" else list(range(self.w.batch))

    def append_to(self, targets: np.ndarray, chunk: int = 8192):
        """Append rows until sequence b holds targets[b] tokens."""
        w = self.w
        writers = self._writers()
        while True:
            new = np.zeros(w.batch, dtype=np.int32)
            for b in writers:
                new[b] = max(0, min(chunk, int(targets[b]) - int(self.cached[b])))
            if not new.any():
                break
            ks, vs = [], []
            for b in range(w.batch):
                if new[b]:
                    k, v = I.kv_rows(w, b, int(self.cached[b]), int(self.cached[b] + new[b]))
                    ks.append(k)
                    vs.append(v)
            k = torch.from_numpy(np.concatenate(ks)).to(torch_dtype(w)).to(self.dev)
            v = torch.from_numpy(np.concatenate(vs)).to(torch_dtype(w)).to(self.dev)
            new_d = torch.from_numpy(new).to(self.dev)
            before = torch.from_numpy(self.cached.copy()).to(self.dev)
            Q.dqk_append(self.desc, k, v, lib_dtype(w), w.batch, new_d, before, int(new.max()),
                         self.table_dev, self.max_pages)
            self.cached += new
        torch.cuda.synchronize(self.dev)

    def prefill(self):
        """Cache every row except the ``append_new`` tail."""
        self.append_to(np.maximum(self.lens - self.w.append_new, 0))

    def append_tail(self):
        self.append_to(self.lens)

    def decode(self, pct: int | None = None, step: int = 0, lens=None, q=None):
        w = self.w
        if self.w.append_new and (self.cached < self.lens)[self._writers()].any():
            self.append_tail()
        pct = w.pct if pct is None else pct
        lens = self.lens if lens is None else np.asarray(lens, dtype=np.int32)
        if q is None:
            q = I.queries(w, np.maximum(lens, 1), step)
        self.q_host = q
        qd = torch.from_numpy(q).to(torch_dtype(w)).to(self.dev)
        keep = O.n_keep(w.d, pct)
        out = torch.empty((w.batch, w.hq, w.d), dtype=torch.float32, device=self.dev)
        sel = torch.full((w.batch, w.hq, keep), -1, dtype=torch.int16, device=self.dev)
        lens_d = torch.from_numpy(lens).to(self.dev)
        Q.dqk_decode(self.desc, qd, lib_dtype(w), w.batch, lens_d, self.table_dev, self.max_pages, pct,
                     out, sel, self.ws, self.ws_bytes)
        torch.cuda.synchronize(self.dev)
        return out.cpu().numpy().astype(np.float64), sel.cpu().numpy()

    def pool_host(self) -> np.ndarray:
        torch.cuda.synchronize(self.dev)
        return self.pool.cpu().numpy().reshape(self.num_pages, self.w.hkv, self.block_bytes)


# ---------------------------------------------------------------------------
# layout decoder, written from the block layout documented in dualqk.h
# ---------------------------------------------------------------------------
def _layout(d, v_ch0, gs=32):
    ng = d // gs                     # scale groups per token
    kc = 0
    ks = 4 * d
    km = ks + 32 * ng
    k0 = km + 32 * ng
    vc = k0 + 32
    vs = vc + 4 * d
    vm = vs + 32 * ng
    v0 = vm + 32 * ng
    return dict(ng=ng, kc=kc, ks=ks, km=km, k0=k0, vc=vc, vs=vs, vm=vm, v0=v0,
                bytes=v0 + (32 if v_ch0 else 0))


def _code_tables(d):
    """(word index, bit) of every (slot t, channel c) for K and for V."""
    ng = d // 32
    kw = np.zeros((16, d), np.int64)
    kb = np.zeros((16, d), np.int64)
    vw = np.zeros((16, d), np.int64)
    vb = np.zeros((16, d), np.int64)
    for t in range(16):
        for c in range(d):
            g, cc = c // 32, c % 32
            r = 2 * (cc // 16) + t // 8
            lane = 4 * (t % 8) + (cc % 16) // 4
            j = cc % 4
            kw[t, c] = lane * ng + r % ng
            kb[t, c] = 8 * j + 2 * (g + ng * (r // ng))
            m, cr, tb, tig, e = c // 16, (c % 16) // 8, t // 8, (t % 8) // 2, t % 2
            lane = 4 * (c % 8) + tig
            if ng == 4:
                vw[t, c] = lane * ng + cr + 2 * tb
                vb[t, c] = 16 * e + 2 * m
            else:
                q = (2 * m + cr) * 2 + tb
                vw[t, c] = lane * ng + q // 8
                vb[t, c] = 16 * e + 2 * (q % 8)
    return kw, kb, vw, vb


def decode_pool(pool: np.ndarray, table_row: np.ndarray, L: int, d: int, v_ch0: int, gs: int = 32) -> O.Cache:
    """Plain arrays (same form as oracle.append) of tokens 0..L-1 of one sequence."""
    lay = _layout(d, v_ch0, gs)
    ng = lay["ng"]
    hkv = pool.shape[1]
    t = np.arange(L)
    slot = t % 16
    blocks = pool[table_row[t // 16]]                       # [L][hkv][bytes]
    w32 = blocks.view(np.uint32)
    w16 = blocks.view(np.uint16)
    kw, kb, vw, vb = _code_tables(d)
    ti = t[:, None, None]
    ji = np.arange(hkv)[None, :, None]
    out = O.Cache()
    out["kcodes"] = ((w32[ti, ji, (lay["kc"] // 4 + kw[slot])[:, None, :]] >> kb[slot][:, None, :]) & 3).astype(np.uint8)
    out["vcodes"] = ((w32[ti, ji, (lay["vc"] // 4 + vw[slot])[:, None, :]] >> vb[slot][:, None, :]) & 3).astype(np.uint8)
    g = np.arange(ng)[None, None, :]
    s = slot[:, None, None]
    kidx = s * ng + g
    vidx = 2 * (ng * (s // 2) + g) + s % 2
    out["kscale"] = w16[ti, ji, lay["ks"] // 2 + kidx]
    out["kmin"] = w16[ti, ji, lay["km"] // 2 + kidx]
    out["vscale"] = w16[ti, ji, lay["vs"] // 2 + vidx]
    out["vmin"] = w16[ti, ji, lay["vm"] // 2 + vidx]
    out["kch0"] = w16[t[:, None], np.arange(hkv)[None, :], lay["k0"] // 2 + (2 * (slot % 8) + slot // 8)[:, None]]
    if v_ch0:
        out["vch0"] = w16[t[:, None], np.arange(hkv)[None, :], lay["v0"] // 2 + slot[:, None]]
    else:
        out["vch0"] = np.zeros((L, hkv), np.uint16)
    return out


# ---------------------------------------------------------------------------
# oracle side
# ---------------------------------------------------------------------------
def oracle_cache(w: I.Workload, b: int, L: int, heads=None) -> O.Cache:
    tk, _, _, _ = workload_transforms(w)
    k, v = I.kv_rows(w, b, 0, L)
    if heads is not None:
        k, v, tk = k[:, heads], v[:, heads], tk[heads]
    return O.append(tk, np.ascontiguousarray(k), np.ascontiguousarray(v), v_ch0=bool(w.v_ch0_protect),
                    gs=w.group_size)


def oracle_reference(w: I.Workload, run: DeviceRun, pct: int | None = None, lens=None) -> dict:
    pct = w.pct if pct is None else pct
    lens = run.lens if lens is None else np.asarray(lens)
    _, tq, _, _ = workload_transforms(w)
    outs, sels, caches = [], [], []
    shared = w.page_order == "shared"
    base = oracle_cache(w, 0, int(lens.max())) if shared else None
    for b in range(w.batch):
        L = int(lens[b])
        cache = base if shared else oracle_cache(w, b, L)
        caches.append(cache)
        o, s, _ = O.decode_seq(cache, run.q_host[b], tq, w.hq, pct, v_ch0=bool(w.v_ch0_protect), L=L)
        outs.append(o)
        sels.append(s)
    return {"out": np.stack(outs), "sel": np.stack(sels), "caches": caches, "lens": lens}


def assert_cache_matches_oracle(run: DeviceRun, ref: dict):
    pool = run.pool_host()
    w = run.w
    for b in range(w.batch):
        L = int(ref["lens"][b])
        if L == 0:
            continue
        got = decode_pool(pool, run.table[b], L, w.d, w.v_ch0_protect, w.group_size)
        exp = ref["caches"][b]
        for key in ("kcodes", "kscale", "kmin", "kch0", "vcodes", "vscale", "vmin", "vch0"):
            e = exp[key][:L]
            if key == "vch0" and not w.v_ch0_protect:
                continue
            if not np.array_equal(got[key], e):
                bad = np.argwhere(got[key] != e)
                raise AssertionError(f"seq {b} {key}: {len(bad)} mismatches, first at {bad[0].tolist()}: "
                                     f"gpu {got[key][tuple(bad[0])]} oracle {e[tuple(bad[0])]}")


def assert_outputs_close(out: np.ndarray, ref: np.ndarray, atol: float = ATOL, rtol_row: float = RTOL_ROW):
    err = np.abs(out - ref)
    num = np.linalg.norm((out - ref).reshape(-1, out.shape[-1]), axis=1)
    den = np.linalg.norm(ref.reshape(-1, ref.shape[-1]), axis=1)
    rel = num / np.maximum(den, 1e-30)
    ok = den > 0
    worst_abs = float(np.nanmax(err)) if err.size else 0.0
    worst_rel = float(np.nanmax(rel[ok])) if ok.any() else 0.0
    name = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    PARITY_RECORDS.append((name, worst_abs, worst_rel))
    print(f"[parity] max abs err {worst_abs:.3e}, max row rel err {worst_rel:.3e}")
    assert np.isfinite(out).all(), "non-finite outputs"
    assert err.max() <= atol, f"max abs error {err.max():.3e} > {atol}"
    if ok.any():
        assert rel[ok].max() <= rtol_row, f"row relative error {rel[ok].max():.3e} > {rtol_row}"
    return worst_abs, worst_rel
