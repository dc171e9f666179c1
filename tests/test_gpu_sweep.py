"""Parity on the sweep shape at full size: 16 sequences x 128K tokens, 32/8
heads, head_dim 128, random page order, every sparsity of the sweep (0, 20,
40, 60 %).  K/V are drawn on the device (the CPU draw of 16 x 128K rows takes
minutes), exactly as the sweep benchmark draws them; the rows of the sampled
(sequence, kv head) units are copied back and run through the oracle: packed
codes, scales, channel 0 and kept channels bit-exact, outputs within
2e-3 abs / 1e-2 per-row relative.  The sweep's smaller batch and context
points are prefixes of the same cache (batch b, context L use sequences
0..b-1 and their first L tokens) and are checked on one sampled unit each.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import harness as H  # noqa: E402
from bit_kv_cache_dqk_b200 import dualqk as Q  # noqa: E402
from bit_kv_cache_dqk_b200 import inputs as I  # noqa: E402
from oracle import oracle as O  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

UNITS = [(3, 2), (14, 7)]          # (sequence, kv head) compared with the oracle at full size
CHUNK = 4096


@pytest.fixture(scope="module")
def sweep():
    w = I.CONFIGS["sweep"]
    dev = torch.device("cuda", 0)
    B, L = w.batch, w.ctx
    lens = np.full(B, L, np.int32)
    table, num_pages = I.page_table(w, lens)
    tk, tq, _, _ = I.transforms(w)
    t_k, t_q = torch.from_numpy(tk).to(dev), torch.from_numpy(tq).to(dev)
    probe = Q.layer_desc(w.d, w.hq, w.hkv, 0, 0, 0, 1)
    pool = torch.empty(num_pages * w.hkv * Q.dqk_block_bytes(probe), dtype=torch.uint8, device=dev)
    desc = Q.layer_desc(w.d, w.hq, w.hkv, t_k, t_q, pool, num_pages)
    table_d = torch.from_numpy(table).to(dev)
    keep_rows = {u: ([], []) for u in UNITS}
    new_d = torch.full((B,), CHUNK, dtype=torch.int32, device=dev)
    for t0 in range(0, L, CHUNK):
        k, v = I.kv_rows_device(w, range(B), t0, t0 + CHUNK, dev)
        before = torch.full((B,), t0, dtype=torch.int32, device=dev)
        Q.dqk_append(desc, k, v, Q.DQK_BF16, B, new_d, before, CHUNK, table_d, table.shape[1])
        for (b, j), (ks, vs) in keep_rows.items():
            ks.append(k[b * CHUNK:(b + 1) * CHUNK, j].float().cpu().numpy())
            vs.append(v[b * CHUNK:(b + 1) * CHUNK, j].float().cpu().numpy())
    torch.cuda.synchronize(dev)
    rows = {u: (np.concatenate(ks), np.concatenate(vs)) for u, (ks, vs) in keep_rows.items()}
    q = I.queries(w, lens)
    return dict(w=w, dev=dev, desc=desc, pool=pool, table=table, table_d=table_d, tk=tk, tq=tq, rows=rows, q=q,
                num_pages=num_pages)


def _decode(S, B, L, pct):
    w, dev = S["w"], S["dev"]
    ws_bytes = Q.dqk_decode_workspace_size(S["desc"], B, S["table"].shape[1])
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    keep = O.n_keep(w.d, pct)
    out = torch.empty((B, w.hq, w.d), dtype=torch.float32, device=dev)
    sel = torch.full((B, w.hq, keep), -1, dtype=torch.int16, device=dev)
    qd = torch.from_numpy(S["q"][:B]).to(torch.bfloat16).to(dev)
    lens_d = torch.full((B,), L, dtype=torch.int32, device=dev)
    Q.dqk_decode(S["desc"], qd, Q.DQK_BF16, B, lens_d, S["table_d"], S["table"].shape[1], pct, out, sel, ws,
                 ws_bytes)
    torch.cuda.synchronize(dev)
    assert Q.dqk_last_device_error() == Q.DQK_OK
    return out.cpu().numpy().astype(np.float64), sel.cpu().numpy()


def _check_unit(S, out, sel, b, j, L, pct, check_cache):
    w = S["w"]
    G = w.group
    k, v = S["rows"][(b, j)]
    cache = O.append(S["tk"][j:j + 1], np.ascontiguousarray(k[:L, None, :]), np.ascontiguousarray(v[:L, None, :]))
    if check_cache:
        pool = S["pool"].cpu().numpy().reshape(S["num_pages"], w.hkv, -1)
        got = H.decode_pool(pool[:, j:j + 1], S["table"][b], L, w.d, 0)
        for key in ("kcodes", "kscale", "kmin", "kch0", "vcodes", "vscale", "vmin"):
            assert np.array_equal(got[key], cache[key]), (b, j, key)
    q = S["q"][b, j * G:(j + 1) * G].astype(np.float32)
    o, s, _ = O.decode_seq(cache, q, S["tq"][j:j + 1], G, pct, L=L)
    assert np.array_equal(sel[b, j * G:(j + 1) * G], s)
    H.assert_outputs_close(out[b, j * G:(j + 1) * G], o)


@pytest.mark.parametrize("pct", [0, 20, 40, 60])
def test_sweep_full_size_every_sparsity(sweep, pct):
    w = sweep["w"]
    out, sel = _decode(sweep, w.batch, w.ctx, pct)
    assert np.isfinite(out).all()
    for i, (b, j) in enumerate(UNITS):
        _check_unit(sweep, out, sel, b, j, w.ctx, pct, check_cache=(pct == 0))


@pytest.mark.parametrize("B,L", [(4, 32768), (4, 8192)])
def test_sweep_smaller_points(sweep, B, L):
    out, sel = _decode(sweep, B, L, 40)
    _check_unit(sweep, out, sel, 3, 2, L, 40, check_cache=False)
