"""GPU: dqk_decode_step (append + decode with the two overlapped on the GPU)
gives the same bytes as dqk_append followed by dqk_decode, and matches the
oracle.  Several consecutive one-token steps check that the attention of a
step sees the row its own append wrote."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import harness as H  # noqa: E402
from bit_kv_cache_dqk_b200 import dualqk as Q  # noqa: E402
from bit_kv_cache_dqk_b200 import inputs as I  # noqa: E402
from oracle import oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu


def _rows(w, lo, hi, dev):
    """Rows [lo[b], hi[b]) of every sequence, concatenated in b order."""
    ks, vs = [], []
    for b in range(w.batch):
        if hi[b] > lo[b]:
            k, v = I.kv_rows(w, b, int(lo[b]), int(hi[b]))
            ks.append(k)
            vs.append(v)
    k = torch.from_numpy(np.concatenate(ks)).to(H.torch_dtype(w)).to(dev)
    v = torch.from_numpy(np.concatenate(vs)).to(H.torch_dtype(w)).to(dev)
    return k, v


def _step(run, lo, hi, fused, pct=None):
    w = run.w
    dev = run.dev
    pct = w.pct if pct is None else pct
    k, v = _rows(w, lo, hi, dev)
    new = (hi - lo).astype(np.int32)
    new_d = torch.from_numpy(new).to(dev)
    before = torch.from_numpy(lo.astype(np.int32)).to(dev)
    lens_d = torch.from_numpy(hi.astype(np.int32)).to(dev)
    q = I.queries(w, np.maximum(hi, 1), 0)
    qd = torch.from_numpy(q).to(H.torch_dtype(w)).to(dev)
    keep = O.n_keep(w.d, pct)
    out = torch.empty((w.batch, w.hq, w.d), dtype=torch.float32, device=dev)
    sel = torch.full((w.batch, w.hq, keep), -1, dtype=torch.int16, device=dev)
    if fused:
        Q.dqk_decode_step(run.desc, k, v, H.lib_dtype(w), new_d, before, int(new.max()), qd, H.lib_dtype(w),
                          w.batch, lens_d, run.table_dev, run.max_pages, pct, out, sel, run.ws, run.ws_bytes)
    else:
        Q.dqk_append(run.desc, k, v, H.lib_dtype(w), w.batch, new_d, before, int(new.max()), run.table_dev,
                     run.max_pages)
        Q.dqk_decode(run.desc, qd, H.lib_dtype(w), w.batch, lens_d, run.table_dev, run.max_pages, pct, out, sel,
                     run.ws, run.ws_bytes)
    torch.cuda.synchronize(dev)
    run.cached = hi.astype(np.int32).copy()
    run.q_host = q
    return out.cpu().numpy().astype(np.float64), sel.cpu().numpy()


def test_step_equals_append_then_decode_and_oracle():
    w = I.CONFIGS["llama"].with_(name="llama-step", batch=5, ctx=None, ctx_lo=20, ctx_hi=900, page_order="random")
    lens = I.lengths(w)
    new = np.array([1, 16, 17, 3, 40], dtype=np.int32)   # crosses page boundaries
    lo = lens - new
    a, b = H.DeviceRun(w, lens=lens), H.DeviceRun(w, lens=lens)
    a.append_to(lo)
    b.append_to(lo)
    oa, sa = _step(a, lo, lens, fused=True)
    ob, sb = _step(b, lo, lens, fused=False)
    assert np.array_equal(sa, sb) and np.array_equal(oa, ob)
    assert np.array_equal(a.pool_host(), b.pool_host())
    ref = H.oracle_reference(w, a)
    H.assert_cache_matches_oracle(a, ref)
    assert np.array_equal(sa, ref["sel"])
    H.assert_outputs_close(oa, ref["out"])
    assert Q.dqk_last_device_error() == Q.DQK_OK


def test_consecutive_one_token_steps():
    w = I.CONFIGS["llama"].with_(name="llama-steps", batch=4, ctx=None, ctx_lo=30, ctx_hi=400, page_order="random")
    final = I.lengths(w)
    a, b = H.DeviceRun(w, lens=final), H.DeviceRun(w, lens=final)
    start = final - 12
    a.append_to(start)
    b.append_to(start)
    for t in range(12):
        lo, hi = start + t, start + t + 1
        oa, sa = _step(a, lo, hi, fused=True)
        ob, sb = _step(b, lo, hi, fused=False)
        assert np.array_equal(sa, sb) and np.array_equal(oa, ob), f"step {t}"
    ref = H.oracle_reference(w, a)
    H.assert_outputs_close(oa, ref["out"])


def test_step_rejects_bad_arguments_before_launch():
    w = I.CONFIGS["llama"].with_(name="llama-args", batch=2, ctx=64)
    run = H.DeviceRun(w)
    before = run.pool.clone()
    dev = run.dev
    k = torch.zeros((2, w.hkv, w.d), dtype=torch.bfloat16, device=dev)
    new_d = torch.ones(2, dtype=torch.int32, device=dev)
    lens_d = torch.full((2,), 64, dtype=torch.int32, device=dev)
    q = torch.zeros((2, w.hq, w.d), dtype=torch.bfloat16, device=dev)
    out = torch.empty((2, w.hq, w.d), dtype=torch.float32, device=dev)
    # valid append part, invalid decode part (sparsity 100): nothing may run
    st = Q.dqk_decode_step(run.desc, k, k, Q.DQK_BF16, new_d, lens_d - 1, 1, q, Q.DQK_BF16, 2, lens_d,
                           run.table_dev, run.max_pages, 100, out, None, run.ws, run.ws_bytes,
                           raise_on_error=False)
    assert st == Q.DQK_ERR_INVALID_ARG
    torch.cuda.synchronize(dev)
    assert torch.equal(run.pool, before)
