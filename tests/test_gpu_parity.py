"""GPU parity: libdualqk (through the C ABI) against the CPU oracle.

Bit-exact: packed codes, fp16 scales/mins, BF16 channel 0, selected channel
indices.  Outputs: max abs error <= 2e-3 and per-row relative error <= 1e-2.
Small cases run the oracle on everything (several pages, ragged tails);
the full-size workloads are checked on sampled (sequence, kv head) units.
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

pytestmark = pytest.mark.gpu


def small(name, **kw):
    return I.CONFIGS[name].with_(name=f"{name}-small", **kw)


CASES = {
    # config 1 exactly as specified (fp32 K/V, d=64, 4 queries sharing pages)
    "tiny": I.CONFIGS["tiny"],
    # llama layer, ragged lengths incl. 1, 15, 16, 17 tokens, random page order
    "llama-ragged": small("llama", batch=6, ctx=None, ctx_lo=1, ctx_hi=1100, page_order="random"),
    # qwen layer: heavy-tailed keys, 64 appended rows on top of the prefill
    "qwen-small": small("qwen", batch=3, ctx_lo=100, ctx_hi=700),
    # value channel 0 protected as well
    "vch0": small("llama", batch=2, ctx=333, v_ch0_protect=1),
    # MHA and other group ratios
    "g1-d128": small("llama", batch=2, hq=4, hkv=4, ctx=257),
    "g2-d64": small("llama", batch=2, hq=8, hkv=4, d=64, ctx=500),
    "g8": small("llama", batch=2, hq=16, hkv=2, ctx=600),
    # one (scale, min) group per token (74 B per token and kv head), ragged, random pages
    "g128": small("llama", batch=4, ctx=None, ctx_lo=1, ctx_hi=700, page_order="random", group_size=128),
    "g128-vch0": small("llama", batch=2, ctx=333, v_ch0_protect=1, group_size=128),
    "g64-d64": small("llama", batch=2, hq=8, hkv=4, d=64, ctx=500, group_size=64),
    # calibrated transform pair and structured queries (next-step row f1)
    "calibrated": small("llama_cal", batch=2, ctx=None, ctx_lo=300, ctx_hi=900),
    # lengths that are whole pages: run boundaries fall at every offset within a
    # warp's four pages of a stage with the run's last page full, so the pages on
    # each side of a boundary are consumed as separate batches
    "full-pages": small("llama", batch=12, ctx=None, ctx_lo=16, ctx_hi=900, len_multiple=16, page_order="random"),
    # five kv heads: one head per chunk, the most pages per stage; long enough
    # that every CTA's ring wraps several times
    "hkv5-wrap": small("llama", batch=2, hq=20, hkv=5, ctx=34000, page_order="random"),
}


@pytest.mark.parametrize("case", list(CASES))
def test_append_and_decode_match_oracle(case):
    w = CASES[case]
    run = H.DeviceRun(w)
    run.prefill()
    out, sel = run.decode()
    ref = H.oracle_reference(w, run)
    H.assert_cache_matches_oracle(run, ref)
    assert np.array_equal(sel, ref["sel"])
    H.assert_outputs_close(out, ref["out"])
    assert Q.dqk_last_device_error() == Q.DQK_OK


@pytest.mark.parametrize("pct", [0, 20, 60, 99])
def test_sparsity_levels(pct):
    w = small("llama", batch=2, ctx=700)
    run = H.DeviceRun(w)
    run.prefill()
    out, sel = run.decode(pct=pct)
    ref = H.oracle_reference(w, run, pct=pct)
    assert np.array_equal(sel, ref["sel"])
    H.assert_outputs_close(out, ref["out"])


def test_zero_and_one_token_contexts():
    w = small("llama", batch=3, ctx=40)
    run = H.DeviceRun(w)
    run.prefill()
    lens = np.array([0, 1, 40], dtype=np.int32)
    out, sel = run.decode(lens=lens)
    assert np.all(out[0] == 0.0)
    ref = H.oracle_reference(w, run, lens=lens)
    H.assert_outputs_close(out[1:], ref["out"][1:])
    assert np.array_equal(sel, ref["sel"])


def test_incremental_appends_equal_one_shot():
    """Appending row by row (decode steps) packs the same bytes as one call."""
    w = small("llama", batch=2, ctx=70, page_order="random")
    a = H.DeviceRun(w)
    a.prefill()
    b = H.DeviceRun(w)
    for L in [1, 2, 15, 16, 17, 33, 69, 70]:
        b.append_to(np.full(w.batch, L))
    assert np.array_equal(a.pool_host()[a.table[:, :5].ravel()], b.pool_host()[b.table[:, :5].ravel()])


def test_split_results_independent_of_page_placement():
    """Same rows, different physical page order: identical outputs."""
    w = small("llama", batch=2, ctx=900, page_order="random")
    a = H.DeviceRun(w)
    a.prefill()
    oa, sa = a.decode()
    w2 = w.with_(page_order="sequential")
    b = H.DeviceRun(w2)
    b.prefill()
    ob, sb = b.decode()
    assert np.array_equal(sa, sb) and np.array_equal(oa, ob)


def test_out_of_range_page_id_is_reported_not_faulted():
    w = small("llama", batch=2, ctx=100)
    run = H.DeviceRun(w)
    run.prefill()
    bad = run.table.copy()
    bad[1, 2] = run.num_pages + 7
    run.table_dev = torch.from_numpy(bad).to(run.dev)
    out, _ = run.decode()
    assert Q.dqk_last_device_error() == Q.DQK_ERR_DEVICE_BOUNDS
    assert np.isfinite(out).all()
    assert Q.dqk_last_device_error() == Q.DQK_OK        # the word was cleared


def test_invalid_arguments_are_rejected_before_launch():
    w = small("llama", batch=1, ctx=16)
    run = H.DeviceRun(w)
    st = Q.dqk_decode(run.desc, None, Q.DQK_BF16, 1, run.table_dev, run.table_dev, run.max_pages, 40,
                      None, None, run.ws, run.ws_bytes, raise_on_error=False)
    assert st == Q.DQK_ERR_INVALID_ARG
    st = Q.dqk_decode(run.desc, run.pool, Q.DQK_BF16, 1, run.table_dev, run.table_dev, run.max_pages, 40,
                      run.pool, None, run.ws, 16, raise_on_error=False)
    assert st == Q.DQK_ERR_WORKSPACE_TOO_SMALL


# ---------------------------------------------------------------- full sizes
def _sampled_units(w, run, out, sel, units):
    _, tq, _, _ = H.workload_transforms(w)
    G = w.group
    for b, j in units:
        L = int(run.lens[b])
        cache = H.oracle_cache(w, b, L, heads=[j])
        got = H.decode_pool(run.pool_host()[:, j:j + 1], run.table[b], L, w.d, w.v_ch0_protect, w.group_size)
        for key in ("kcodes", "kscale", "kmin", "kch0", "vcodes", "vscale", "vmin"):
            assert np.array_equal(got[key], cache[key]), (b, j, key)
        o, s, _ = O.decode_seq(cache, run.q_host[b, j * G:(j + 1) * G], tq[j:j + 1], G, w.pct, L=L)
        assert np.array_equal(sel[b, j * G:(j + 1) * G], s)
        H.assert_outputs_close(out[b, j * G:(j + 1) * G], o)


@pytest.mark.slow
@pytest.mark.parametrize("name,units", [("llama", [(0, 0), (7, 5)]),
                                        ("long", [(1, 3), (3, 7)]),
                                        ("long128", [(0, 2), (2, 5)]),
                                        ("qwen", [(2, 1), (15, 6)])])
def test_full_size_configs_sampled(name, units):
    w = I.CONFIGS[name]
    run = H.DeviceRun(w)
    run.prefill()
    out, sel = run.decode()
    assert Q.dqk_last_device_error() == Q.DQK_OK
    assert np.isfinite(out).all()
    _sampled_units(w, run, out, sel, units)
