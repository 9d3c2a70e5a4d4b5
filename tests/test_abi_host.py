"""Host-side checks of libtq (no GPU): the shared library loads and exports every symbol
declared in include/tq.h, its host parameter generator agrees with the float64 oracle,
and argument errors come back as status codes."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import kv_cache_vector_08_b200 as tq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 15
    L = ctypes.CDLL(tq.lib_path())
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


@pytest.mark.parametrize("d,bits,mode", [(3, 3, 0), (16, 3, 0), (64, 4, 0), (64, 3, 1), (128, 4, 0),
                                         (128, 4, 1), (128, 2, 1), (200, 4, 0), (64, 2, 0)])
def test_host_params_match_oracle(d, bits, mode):
    h = tq.host_params(d, bits, 1000 + d + bits, mode)
    o = oracle.make_params(d, bits, 1000 + d + bits, mode)
    assert np.abs(h["Pi"] - o["Pi"]).max() < 1e-10
    assert np.abs(h["Pi"] @ h["Pi"].T - np.eye(d)).max() < 1e-12
    if mode == 0:
        assert np.abs(h["S"] - o["S"]).max() < 1e-12
    assert np.abs(h["centroids"] - o["centroids"]).max() < 1e-10
    assert np.abs(h["boundaries"] - o["boundaries"]).max() < 1e-10
    K = len(h["centroids"])
    assert h["boundaries"][K // 2 - 1] == 0.0          # exact symmetry, like the oracle


@pytest.mark.slow
def test_host_params_match_oracle_d1536():
    h = tq.host_params(1536, 4, 7, 0)
    o = oracle.make_params(1536, 4, 7, 0)
    assert np.abs(h["Pi"] - o["Pi"]).max() < 1e-10
    assert np.abs(h["centroids"] - o["centroids"]).max() < 1e-10


def test_host_params_seed_changes_rotation():
    a = tq.host_params(16, 3, 1, 0)["Pi"]
    b = tq.host_params(16, 3, 2, 0)["Pi"]
    assert np.abs(a - b).max() > 0.1


def test_argument_errors_without_gpu():
    L = tq.lib()
    h = ctypes.c_void_p()
    assert L.tq_init(None, 128, 4, 0, 0) == 1                    # TQ_ERR_INVALID_ARG
    assert L.tq_init(ctypes.byref(h), 2, 4, 0, 0) == 2           # d < 3: unsupported
    assert L.tq_init(ctypes.byref(h), 5000, 4, 0, 0) == 2
    assert L.tq_init(ctypes.byref(h), 128, 6, 0, 0) == 2         # prod bits > 5
    assert L.tq_init(ctypes.byref(h), 128, 1, 0, 0) == 2         # prod bits < 2
    assert L.tq_init(ctypes.byref(h), 128, 5, 0, 1) == 2         # MSE bits > 4
    assert L.tq_init(ctypes.byref(h), 128, 4, 0, 7) == 1         # bad mode
    assert b"bits" in L.tq_last_error() or b"mode" in L.tq_last_error()
    assert L.tq_host_params(2, 3, 0, 0, None, None, None, None) == 2
    assert L.tq_get_info(None, None) == 1
    assert L.tq_quantize_kv(None, None, 0, 0, 0, None, None, None, 0, None) == 1
    assert L.tq_quantize_workspace_size(None, 0, 10, 128) == 0
    assert L.tq_search_topk(None, None, 0, None, 0, 1, None, None, None, 0, None) == 1
    assert L.tq_decode_workspace_size(1, 0, 8, 128, 1, 100) == 0
    assert L.tq_decode_workspace_size(1, 32, 8, 128, 1, 32768) > 0
    L.tq_free(None)                                              # NULL is ignored


def test_decode_workspace_grows_with_context():
    small = tq.decode_workspace_size(1, 32, 8, 128, 1, 1024)
    big = tq.decode_workspace_size(1, 32, 8, 128, 1, 131072)
    assert 0 < small < big


def test_channel_perm_by_score_puts_the_highest_scores_first():
    score = np.array([0.1, 5.0, 0.2, 5.0, 9.0, 0.0, 0.3, 7.0], dtype=np.float32)
    perm = tq.channel_perm_by_score(score, 4)
    # top 4: channels 4 (9), 7 (7), 1 and 3 (5, ties to the lower channel) -> ascending
    assert perm.tolist() == [1, 3, 4, 7, 0, 2, 5, 6]
    assert sorted(perm.tolist()) == list(range(8))
    assert tq.channel_perm_by_score(score, 0).tolist() == list(range(8))
    with pytest.raises(tq.TQError):
        tq.channel_perm_by_score(score, 9)
