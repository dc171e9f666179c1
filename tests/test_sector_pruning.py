"""How many key-code bytes query-channel pruning could leave unread, CPU only.

"How does Dual-QK compress KV caches to 2-bit while keeping accuracy at 128K
context?", section "Why the cache becomes a bottleneck": the decode reads only
the key channels its pruned query keeps.  With grouped-query attention one
cached key row serves the G query heads of its kv head, so a channel can be
left unread only when none of the G heads keeps it; and DRAM moves whole
32-byte sectors, which in a channel-major code layout (16 tokens x 2 bits per
channel) hold 8 channels.  These tests take the oracle's selections on the
`long` (synthetic whitening pair) and `llama_cal` (calibrated pair, low-rank
queries) workloads and count the 8-channel sectors that no head of a group
keeps.  The fraction stays far below the 10 % of key-code bytes for which a
sector-skipping layout would pay (the block layout here copies whole blocks).
"""
import numpy as np
import pytest

from bit_kv_cache_dqk_b200 import calibrate as Cb
from bit_kv_cache_dqk_b200 import inputs as I
from oracle import oracle as O

SECTOR = 8   # channels of 16 tokens x 2 bits in one 32-byte sector


def _unkept(wl: str, pct: int, n_seq: int = 16):
    """Per (sequence, kv head): channels kept by some head of the group, and
    8-channel sectors kept by none."""
    w = I.CONFIGS[wl]
    _, tq32, _, _ = Cb.layer_transforms(w)
    lens = I.lengths(w)
    kept, empty = [], []
    for step in range(max(1, n_seq // w.batch)):
        q = I.queries(w, lens, step)
        for b in range(w.batch):
            for j in range(w.hkv):
                keep = np.zeros(w.d, bool)
                for h in range(j * w.group, (j + 1) * w.group):
                    _, sel = O.qprep(tq32[j], q[b, h], pct)
                    keep[sel] = True
                kept.append(int(keep.sum()))
                empty.append(int((~keep.reshape(-1, SECTOR).any(axis=1)).sum()))
    return np.array(kept), np.array(empty), w.d // SECTOR


@pytest.mark.parametrize("wl", ["long", "llama_cal"])
def test_no_sector_is_skippable_at_40_percent(wl):
    kept, empty, nsec = _unkept(wl, 40)
    assert kept.min() >= 0.85 * 128          # the group's union covers most channels
    assert empty.sum() == 0                   # every sector holds a kept channel


@pytest.mark.parametrize("wl", ["long", "llama_cal"])
def test_skippable_sectors_stay_below_ten_percent_at_60_percent(wl):
    kept, empty, nsec = _unkept(wl, 60)
    frac = empty.mean() / nsec
    assert frac < 0.10, f"{wl}: {100 * frac:.2f} % of key-code sectors unkept"
    # the union still shrinks with the sparsity
    assert kept.mean() < _unkept(wl, 40)[0].mean()
