"""dqk_decode_noalloc: the decode for callers that cannot allocate device
memory while decoding (plugin hosts whose op interface offers no scratch
buffer, serving loops that forbid allocation after warm-up).  It must give
what dqk_decode gives with a caller workspace, call after call, although all
calls share one static scratch array.

This file is collected last on purpose: it passes alone in a fresh process
and after every other test.
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


def test_noalloc_decode_matches_workspace_decode_on_consecutive_calls():
    w = I.CONFIGS["llama"].with_(name="noalloc", batch=3, ctx=None, ctx_lo=1, ctx_hi=900,
                                 page_order="random")
    run = H.DeviceRun(w)
    run.prefill()
    ref_out, ref_sel = run.decode()                      # dqk_decode with a caller workspace
    assert run.ws_bytes <= Q.DQK_NOALLOC_WORKSPACE_BYTES
    qd = torch.from_numpy(run.q_host).to(H.torch_dtype(w)).to(run.dev)
    lens = torch.from_numpy(run.lens).to(run.dev)
    keep = ref_sel.shape[-1]
    for _ in range(2):                                   # the second call sees the first call's scratch
        out = torch.full((w.batch, w.hq, w.d), float("nan"), dtype=torch.float32, device=run.dev)
        sel = torch.full((w.batch, w.hq, keep), -1, dtype=torch.int16, device=run.dev)
        st = Q.dqk_decode_noalloc(run.desc, qd, H.lib_dtype(w), w.batch, lens, run.table_dev,
                                  run.max_pages, w.pct, out, sel)
        assert st == Q.DQK_OK
        torch.cuda.synchronize(run.dev)
        assert np.array_equal(sel.cpu().numpy(), ref_sel)
        H.assert_outputs_close(out.cpu().numpy().astype(np.float64), ref_out)
    assert Q.dqk_last_device_error() == Q.DQK_OK


def test_noalloc_rejects_requests_beyond_its_scratch():
    w = I.CONFIGS["llama"].with_(name="noalloc-big", batch=1, ctx=16)
    run = H.DeviceRun(w)
    batch = 4096                                         # query-prep scratch alone exceeds 8 MiB
    assert Q.dqk_decode_workspace_size(run.desc, batch, run.max_pages) > Q.DQK_NOALLOC_WORKSPACE_BYTES
    st = Q.dqk_decode_noalloc(run.desc, run.pool, Q.DQK_BF16, batch, run.table_dev, run.table_dev,
                              run.max_pages, 40, run.pool, None, raise_on_error=False)
    assert st == Q.DQK_ERR_WORKSPACE_TOO_SMALL
