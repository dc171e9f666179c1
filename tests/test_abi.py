"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/dualqk.h declares, sizes blocks and workspaces by the
compression formula, and rejects bad arguments before touching a device."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def Q():
    from bit_kv_cache_dqk_b200 import build
    build.build()
    from bit_kv_cache_dqk_b200 import dualqk
    return dualqk


def header_functions():
    text = open(os.path.join(ROOT, "include", "dualqk.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dqk_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_function_is_exported(Q):
    names = header_functions()
    assert len(names) >= 9
    lib = C.CDLL(Q.library_path())
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(Q.EXPORTED) == names


@pytest.mark.parametrize("d,vch0,bytes_", [(128, 0, 1568), (64, 0, 800), (128, 1, 1600), (64, 1, 832)])
def test_block_bytes_follow_compression_formula(Q, d, vch0, bytes_):
    """Per token and kv head: d/4 bytes of K codes + d/4 of V codes (2 bits per
    value), 4 bytes of fp16 (scale, min) per 32-channel group for K and for V,
    2 bytes of BF16 key channel 0 (+2 with value channel 0)."""
    per_token = d // 4 + d // 4 + 2 * 4 * (d // 32) + 2 + 2 * vch0
    desc = Q.layer_desc(d, 8, 2, 0, 0, 0, 1, v_ch0_protect=vch0)
    assert Q.dqk_block_bytes(desc) == 16 * per_token == bytes_
    assert Q.dqk_block_bytes(desc) % 16 == 0


def test_compression_ratio_vs_bf16(Q):
    desc = Q.layer_desc(128, 32, 8, 0, 0, 0, 1)
    per_token = Q.dqk_block_bytes(desc) / 16
    assert per_token == 98
    assert abs(2 * 2 * 128 / per_token - 5.224) < 1e-3       # K+V BF16 = 512 B


@pytest.mark.parametrize("d,vch0,bytes_", [(128, 0, 1184), (64, 0, 672), (128, 1, 1216)])
def test_one_group_per_token_bytes(Q, d, vch0, bytes_):
    """group_size = head_dim: one fp16 (scale, min) per token for K and for V."""
    per_token = d // 4 + d // 4 + 2 * 4 + 2 + 2 * vch0
    desc = Q.layer_desc(d, 8, 2, 0, 0, 0, 1, v_ch0_protect=vch0, group_size=d)
    assert Q.dqk_block_bytes(desc) == 16 * per_token == bytes_


def test_one_group_compression_matches_the_pages(Q):
    """74 B per token and kv head at d = 128: 512/74 = 6.92x against BF16 K+V
    (the 6.8x of "Results at 128K context"); dropping 40 % of the key codes
    from reads leaves 74 - 0.4 * 31.75 = 61.3 B, 8.35x (the estimated 8.3x)."""
    desc = Q.layer_desc(128, 32, 8, 0, 0, 0, 1, group_size=128)
    per_token = Q.dqk_block_bytes(desc) / 16
    assert per_token == 74
    assert abs(512 / per_token - 6.92) < 0.01
    assert abs(512 / (per_token - 0.4 * 127 / 4) - 8.35) < 0.01


def test_unsupported_layers(Q):
    assert Q.dqk_block_bytes(Q.layer_desc(128, 8, 2, 0, 0, 0, 1, group_size=64)) == 0
    assert Q.dqk_block_bytes(Q.layer_desc(96, 8, 2, 0, 0, 0, 1)) == 0
    assert Q.dqk_decode_workspace_size(Q.layer_desc(128, 24, 8, 0, 0, 1, 1), 1, 4) == 0   # G = 3
    assert Q.dqk_decode_workspace_size(Q.layer_desc(128, 32, 8, 0, 0, 0, 1), 1, 4) == 0   # no pool
    assert Q.dqk_decode_workspace_size(Q.layer_desc(128, 32, 8, 0, 0, 256, 1), 4, 8192) > 0


def test_invalid_arguments_rejected_on_host(Q):
    desc = Q.layer_desc(128, 32, 8, 256, 256, 256, 10)
    st = Q.dqk_append(desc, None, 256, Q.DQK_BF16, 1, 256, 256, 1, 256, 1, stream=0, raise_on_error=False)
    assert st == Q.DQK_ERR_INVALID_ARG
    st = Q.dqk_decode(desc, 256, Q.DQK_BF16, 1, 256, 256, 4, 140, 256, None, 256, 1 << 30, stream=0,
                      raise_on_error=False)
    assert st == Q.DQK_ERR_INVALID_ARG                     # sparsity out of range
    st = Q.dqk_decode(desc, 256, Q.DQK_BF16, 1, 256, 256, 4, 40, 256, None, 256, 16, stream=0,
                      raise_on_error=False)
    assert st == Q.DQK_ERR_WORKSPACE_TOO_SMALL
    bad = Q.layer_desc(128, 32, 8, 256, 256, 256, 10, page_size=32)
    st = Q.dqk_decode(bad, 256, Q.DQK_BF16, 1, 256, 256, 4, 40, 256, None, 256, 1 << 30, stream=0,
                      raise_on_error=False)
    assert st == Q.DQK_ERR_UNSUPPORTED


def test_misaligned_transforms_rejected_on_host(Q):
    """The kernels read T_K and T_Q with 16-byte copies: a transform that is not
    16-byte aligned is refused before anything is launched."""
    desc = Q.layer_desc(128, 32, 8, 260, 256, 256, 10)   # T_K 4 bytes off
    st = Q.dqk_append(desc, 256, 256, Q.DQK_BF16, 1, 256, 256, 1, 256, 1, stream=0, raise_on_error=False)
    assert st == Q.DQK_ERR_INVALID_ARG
    desc = Q.layer_desc(128, 32, 8, 256, 264, 256, 10)   # T_Q 8 bytes off
    st = Q.dqk_decode(desc, 256, Q.DQK_BF16, 1, 256, 256, 4, 40, 256, None, 256, 1 << 30, stream=0,
                      raise_on_error=False)
    assert st == Q.DQK_ERR_INVALID_ARG


def test_status_strings(Q):
    assert Q.dqk_status_string(Q.DQK_OK) == "DQK_OK"
    assert Q.dqk_status_string(Q.DQK_ERR_TIMEOUT) == "DQK_ERR_TIMEOUT"
    assert Q.dqk_status_string(77) == "DQK_UNKNOWN_STATUS"
