"""GPU: context-parallel decode through the C ABI.  Each sequence's pages are
split into `world` contiguous ranges (the share each rank would hold);
dqk_decode_partial decodes each range into (m, l, o) records, which are
compared with the oracle's records of the same row range, and
dqk_merge_partials of the stacked records is compared with the oracle's
whole-sequence decode and with the device's own single-range decode."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import harness as H  # noqa: E402
from bit_kv_cache_dqk_b200 import context_parallel as CP  # noqa: E402
from bit_kv_cache_dqk_b200 import dualqk as Q  # noqa: E402
from bit_kv_cache_dqk_b200 import inputs as I  # noqa: E402
from oracle import oracle as O  # noqa: E402

pytestmark = pytest.mark.gpu


def small(name, **kw):
    return I.CONFIGS[name].with_(name=f"{name}-cp", **kw)


CASES = {
    "llama-ragged": small("llama", batch=4, ctx=None, ctx_lo=1, ctx_hi=700, page_order="random"),
    "g8-d128": small("llama", batch=2, hq=16, hkv=2, ctx=900),
    "g2-d64": small("llama", batch=3, hq=8, hkv=4, d=64, ctx=None, ctx_lo=30, ctx_hi=600),
    "g128-calibrated": small("llama_cal", batch=2, ctx=800, group_size=128),
}


def assert_records_match(rec, ref):
    """Records agree up to the choice of m: l 2^m and o 2^m are what is defined."""
    empty = ref[..., 0] == -np.inf
    assert np.all(rec[..., 0][empty] == -np.inf)
    assert np.all(rec[..., 1:][empty] == 0.0)
    r, f = rec[~empty], ref[~empty]
    assert np.isfinite(r).all()
    scale = np.exp2(r[:, 0] - f[:, 0])
    np.testing.assert_allclose(r[:, 1] * scale, f[:, 1], rtol=1e-2)
    H.assert_outputs_close(r[:, 2:] / r[:, 1:2], f[:, 2:] / f[:, 1:2])


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("case", list(CASES))
def test_context_parallel_matches_oracle(case, world):
    w = CASES[case]
    run = H.DeviceRun(w)
    run.prefill()
    full, sel_full = run.decode()
    ref = H.oracle_reference(w, run)
    lens = run.lens
    _, tq, _, _ = H.workload_transforms(w)
    qd = torch.from_numpy(run.q_host).to(H.torch_dtype(w)).to(run.dev)
    keep = O.n_keep(w.d, w.pct)
    parts = []
    for r in range(world):
        sub_lens, sub = CP.rank_view(lens, run.table, r, world)
        part = torch.empty((w.batch, w.hq, w.d + 2), dtype=torch.float32, device=run.dev)
        sel = torch.full((w.batch, w.hq, keep), -1, dtype=torch.int16, device=run.dev)
        Q.dqk_decode_partial(run.desc, qd, H.lib_dtype(w), w.batch, torch.from_numpy(sub_lens).to(run.dev),
                             torch.from_numpy(sub).to(run.dev), sub.shape[1], w.pct, part, sel, run.ws,
                             run.ws_bytes)
        torch.cuda.synchronize(run.dev)
        assert Q.dqk_last_device_error() == Q.DQK_OK
        np.testing.assert_array_equal(sel.cpu().numpy(), ref["sel"])
        rec = part.cpu().numpy().astype(np.float64)
        for b in range(w.batch):
            p0, _ = CP.page_range((int(lens[b]) + CP.PAGE - 1) // CP.PAGE, r, world)
            t0 = p0 * CP.PAGE
            oref = O.decode_partial(ref["caches"][b], run.q_host[b], tq, w.hq, w.pct,
                                    v_ch0=bool(w.v_ch0_protect), t0=t0, t1=t0 + int(sub_lens[b]))
            assert_records_match(rec[b], oref)
        parts.append(part)
    out = torch.empty((w.batch, w.hq, w.d), dtype=torch.float32, device=run.dev)
    Q.dqk_merge_partials(torch.stack(parts), world, w.batch, w.hq, w.d, out)
    torch.cuda.synchronize(run.dev)
    merged = out.cpu().numpy().astype(np.float64)
    H.assert_outputs_close(merged, ref["out"])
    # each split rounds its softmax weights to fp16 against its own running
    # max, so two partitions of the same pages agree to ~2^-11 of |v|, not bitwise
    np.testing.assert_allclose(merged, full, rtol=0, atol=1e-3)


def test_single_range_partial_then_merge_is_decode():
    w = CASES["llama-ragged"]
    run = H.DeviceRun(w)
    run.prefill()
    full, _ = run.decode()
    qd = torch.from_numpy(run.q_host).to(H.torch_dtype(w)).to(run.dev)
    keep = O.n_keep(w.d, w.pct)
    part = torch.empty((w.batch, w.hq, w.d + 2), dtype=torch.float32, device=run.dev)
    sel = torch.empty((w.batch, w.hq, keep), dtype=torch.int16, device=run.dev)
    Q.dqk_decode_partial(run.desc, qd, H.lib_dtype(w), w.batch, torch.from_numpy(run.lens).to(run.dev),
                         run.table_dev, run.max_pages, w.pct, part, sel, run.ws, run.ws_bytes)
    out = torch.empty((w.batch, w.hq, w.d), dtype=torch.float32, device=run.dev)
    Q.dqk_merge_partials(part, 1, w.batch, w.hq, w.d, out)
    torch.cuda.synchronize(run.dev)
    # the same split-K partitions and combine order as dqk_decode, then one exact division
    np.testing.assert_allclose(out.cpu().numpy(), full, rtol=1e-6, atol=1e-7)


def test_all_empty_ranges_merge_to_zero():
    w = CASES["g2-d64"]
    run = H.DeviceRun(w)
    run.prefill()
    run.decode()
    qd = torch.from_numpy(run.q_host).to(H.torch_dtype(w)).to(run.dev)
    zero = torch.zeros(w.batch, dtype=torch.int32, device=run.dev)
    part = torch.full((w.batch, w.hq, w.d + 2), 7.0, dtype=torch.float32, device=run.dev)
    sel = torch.empty((w.batch, w.hq, O.n_keep(w.d, w.pct)), dtype=torch.int16, device=run.dev)
    Q.dqk_decode_partial(run.desc, qd, H.lib_dtype(w), w.batch, zero, run.table_dev, run.max_pages, w.pct,
                         part, sel, run.ws, run.ws_bytes)
    rec = part.cpu().numpy()
    assert np.all(rec[..., 0] == -np.inf) and np.all(rec[..., 1:] == 0.0)
    out = torch.full((w.batch, w.hq, w.d), 7.0, dtype=torch.float32, device=run.dev)
    Q.dqk_merge_partials(torch.stack([part, part]), 2, w.batch, w.hq, w.d, out)
    assert np.all(out.cpu().numpy() == 0.0)


def test_merge_rejects_bad_arguments():
    buf = torch.zeros(4 * 130, dtype=torch.float32, device="cuda:0")
    out = torch.zeros(4 * 128, dtype=torch.float32, device="cuda:0")
    assert Q.dqk_merge_partials(buf, 0, 1, 4, 128, out, raise_on_error=False) == Q.DQK_ERR_INVALID_ARG
    assert Q.dqk_merge_partials(buf, 1, 1, 4, 96, out, raise_on_error=False) == Q.DQK_ERR_UNSUPPORTED
