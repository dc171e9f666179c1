"""GPU: the BF16 comparison decode (dqk_bf16_append / dqk_bf16_decode) against
textbook softmax attention from the oracle (quantization off, identity
transforms, every channel kept, fp64) on the same BF16 K/V values."""
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
    return I.CONFIGS[name].with_(name=f"{name}-b16", **kw)


CASES = {
    "tiny": I.CONFIGS["tiny"],
    "llama-ragged": small("llama", batch=5, ctx=None, ctx_lo=1, ctx_hi=900, page_order="random"),
    "g1-d128": small("llama", batch=2, hq=4, hkv=4, ctx=257),
    "g2-d64": small("llama", batch=2, hq=8, hkv=4, d=64, ctx=500),
    "g8": small("llama", batch=2, hq=16, hkv=2, ctx=600),
    "qwen-small": small("qwen", batch=3, ctx_lo=100, ctx_hi=700),
}


class Bf16Run:
    def __init__(self, w, lens=None, device="cuda:0"):
        self.w = w
        self.dev = torch.device(device)
        self.lens = I.lengths(w) if lens is None else np.asarray(lens, np.int32)
        self.table, self.num_pages = I.page_table(w, np.maximum(self.lens, 1))
        self.max_pages = self.table.shape[1]
        probe = Q.layer_desc(w.d, w.hq, w.hkv, 0, 0, 0, 1)
        self.bb = Q.dqk_bf16_block_bytes(probe)
        self.pool = torch.full((self.num_pages * w.hkv * self.bb,), 0xFF, dtype=torch.uint8, device=self.dev)
        self.desc = Q.layer_desc(w.d, w.hq, w.hkv, 0, 0, self.pool, self.num_pages)
        self.table_dev = torch.from_numpy(self.table).to(self.dev)
        self.cached = np.zeros(w.batch, np.int32)
        self.ws_bytes = Q.dqk_bf16_decode_workspace_size(self.desc, w.batch, self.max_pages)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.dev)

    def writers(self):
        return [0] if self.w.page_order == "shared" else list(range(self.w.batch))

    def append_to(self, targets, chunk=4096):
        w = self.w
        while True:
            new = np.zeros(w.batch, np.int32)
            for b in self.writers():
                new[b] = max(0, min(chunk, int(targets[b]) - int(self.cached[b])))
            if not new.any():
                break
            ks, vs = zip(*[I.kv_rows(w, b, int(self.cached[b]), int(self.cached[b] + new[b]))
                           for b in range(w.batch) if new[b]])
            k = torch.from_numpy(np.concatenate(ks)).to(H.torch_dtype(w)).to(self.dev)
            v = torch.from_numpy(np.concatenate(vs)).to(H.torch_dtype(w)).to(self.dev)
            Q.dqk_bf16_append(self.desc, k, v, H.lib_dtype(w), w.batch, torch.from_numpy(new).to(self.dev),
                              torch.from_numpy(self.cached.copy()).to(self.dev), int(new.max()), self.table_dev,
                              self.max_pages)
            self.cached += new
        torch.cuda.synchronize(self.dev)

    def decode(self, lens=None):
        w = self.w
        lens = self.lens if lens is None else np.asarray(lens, np.int32)
        self.q_host = I.queries(w, np.maximum(lens, 1))
        qd = torch.from_numpy(self.q_host).to(H.torch_dtype(w)).to(self.dev)
        out = torch.empty((w.batch, w.hq, w.d), dtype=torch.float32, device=self.dev)
        Q.dqk_bf16_decode(self.desc, qd, H.lib_dtype(w), w.batch, torch.from_numpy(lens).to(self.dev),
                          self.table_dev, self.max_pages, out, self.ws, self.ws_bytes)
        torch.cuda.synchronize(self.dev)
        return out.cpu().numpy().astype(np.float64)


def bf16_values(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float32).numpy()


def reference(w, q, lens):
    eye = np.broadcast_to(np.eye(w.d), (w.hkv, w.d, w.d)).copy()
    outs = []
    for b in range(w.batch):
        L = int(lens[b])
        src = 0 if w.page_order == "shared" else b
        k, v = I.kv_rows(w, src, 0, L)
        outs.append(O.decode_dense(eye, eye, bf16_values(k), bf16_values(v), q[b], 0))
    return np.stack(outs)


@pytest.mark.parametrize("case", list(CASES))
def test_bf16_decode_matches_textbook_attention(case):
    w = CASES[case]
    run = Bf16Run(w)
    run.append_to(run.lens)
    out = run.decode()
    H.assert_outputs_close(out, reference(w, run.q_host, run.lens))
    assert Q.dqk_last_device_error() == Q.DQK_OK


def test_bf16_zero_and_one_token_and_row_appends():
    w = small("llama", batch=3, ctx=40)
    run = Bf16Run(w)
    for L in [1, 7, 16, 17, 40]:
        run.append_to(np.full(w.batch, L))
    lens = np.array([0, 1, 40], np.int32)
    out = run.decode(lens)
    assert np.all(out[0] == 0.0)
    ref = reference(w.with_(batch=3), run.q_host, np.maximum(lens, 1))
    H.assert_outputs_close(out[1:], ref[1:])


def test_bf16_out_of_range_page_is_reported():
    w = small("llama", batch=2, ctx=100)
    run = Bf16Run(w)
    run.append_to(run.lens)
    bad = run.table.copy()
    bad[0, 3] = run.num_pages + 5
    run.table_dev = torch.from_numpy(bad).to(run.dev)
    out = run.decode()
    assert Q.dqk_last_device_error() == Q.DQK_ERR_DEVICE_BOUNDS
    assert np.isfinite(out).all()
    assert Q.dqk_last_device_error() == Q.DQK_OK
