"""Failure detection on the GPU, without faulting or hanging it.

Every wait of the decode kernel is bounded.  The test-only entry point
dqk_test_decode_stall makes one of them run out on purpose: the producer warp
of CTA 0 never arms its second ring stage and the ring waits give up after
1 ms.  The consumers of that CTA stop, the producer drains the copies it had
issued, every CTA still takes part in both grid barriers, the launch ends,
and the device error word reads DQK_ERR_TIMEOUT.  Nothing stays in flight:
the next normal decode in the same process is exact again.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import harness as H  # noqa: E402
from bit_kv_cache_dqk_b200 import dualqk as Q  # noqa: E402
from bit_kv_cache_dqk_b200 import inputs as I  # noqa: E402

pytestmark = pytest.mark.gpu


def test_stalled_stage_reports_timeout_and_next_decode_is_exact():
    # long enough that CTA 0 has more than two ring stages of pages
    w = I.CONFIGS["llama"].with_(name="stall", batch=2, ctx=20000, page_order="random")
    run = H.DeviceRun(w)
    run.prefill()
    ref_out, ref_sel = run.decode()
    assert Q.dqk_last_device_error() == Q.DQK_OK
    qd = torch.from_numpy(run.q_host).to(H.torch_dtype(w)).to(run.dev)
    lens = torch.from_numpy(run.lens).to(run.dev)
    out = torch.empty((w.batch, w.hq, w.d), dtype=torch.float32, device=run.dev)
    sel = torch.empty_like(torch.from_numpy(ref_sel)).to(run.dev)
    st = Q.dqk_test_decode_stall(run.desc, qd, H.lib_dtype(w), w.batch, lens, run.table_dev, run.max_pages, w.pct,
                                 out, sel, run.ws, run.ws_bytes)
    assert st == Q.DQK_OK                                 # the launch itself is fine
    assert Q.dqk_last_device_error() == Q.DQK_ERR_TIMEOUT   # the bounded wait ran out
    assert Q.dqk_last_device_error() == Q.DQK_OK            # and the word was cleared
    for _ in range(2):                                      # the context and the library are intact
        out2, sel2 = run.decode()
        assert Q.dqk_last_device_error() == Q.DQK_OK
        assert np.array_equal(sel2, ref_sel)
        assert np.array_equal(out2, ref_out)
