"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, its host-side time-bucket table agrees with the oracle, and
invalid arguments are rejected on the host before any device work."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import hstu as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hstu.h")


@pytest.fixture(scope="module")
def H():
    from hstu_sequential_transduction_jagged_b200 import build, hstu
    build.build()
    return hstu


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s+(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if not n.startswith("HSTU_")))


def test_header_declares_entry_points():
    names = declared_functions()
    for must in ("hstu_attn_fwd", "hstu_layer_fwd", "mfalcon_score", "hstu_forward"):
        assert must in names


def test_library_exports_every_declared_symbol(H):
    L = H.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in H.EXPORTS, f"binding does not marshal {name}"


@pytest.mark.parametrize("Tb", [1, 2, 32, 128, 256])
def test_threshold_table_matches_oracle(H, Tb):
    thr = H.time_bucket_thresholds(Tb)
    assert np.array_equal(thr, O.time_bucket_thresholds(Tb))
    # each edge separates the oracle's buckets exactly (the oracle evaluates the
    # logarithm itself, so a libm/numpy disagreement at an edge would show here)
    for k in range(1, Tb):
        if thr[k] == np.iinfo(np.int64).max:  # beyond any representable difference
            assert O.time_bucket(1 << 62, 1 << 30) < k
            continue
        assert O.time_bucket(thr[k], Tb) >= k
        if thr[k] > 0:
            assert O.time_bucket(thr[k] - 1, Tb) < k


def _cfg(H, **kw):
    base = dict(d_model=256, num_heads=4, num_pos_buckets=512, num_time_buckets=128)
    base.update(kw)
    return H.LayerConfig(**base)


def test_host_validation_without_device(H):
    L = H.lib()
    good = _cfg(H).c()
    jag = H.JaggedT(2, 10, 8, None, None)  # offsets NULL with batch > 0
    st = L.hstu_attn_fwd(None, ctypes.byref(jag), None, None, None, None, None, None, None, 0, None)
    assert st == 1  # NULL cfg
    st = L.hstu_attn_fwd(ctypes.byref(good), ctypes.byref(jag), None, None, None, None, None,
                         None, None, 0, None)
    assert st == 1  # NULL offsets
    bad = _cfg(H, dqk=32).c()
    ok_jag = H.JaggedT(0, 0, 0, None, None)
    st = L.hstu_attn_fwd(ctypes.byref(bad), ctypes.byref(ok_jag), None, None, None, None, None,
                         None, None, 0, None)
    assert st == 2  # unsupported head width
    long_jag = H.JaggedT(1, 20000, 20000, 16, 16)
    st = L.hstu_attn_fwd(ctypes.byref(good), ctypes.byref(long_jag), None, None, None, None,
                         None, None, None, 0, None)
    assert st == 2  # beyond the longest supported sequence
    neg = H.JaggedT(-1, 0, 0, None, None)
    st = L.hstu_attn_fwd(ctypes.byref(good), ctypes.byref(neg), None, None, None, None, None,
                         None, None, 0, None)
    assert st == 1
    assert L.hstu_time_bucket_thresholds(0, None) == 1
    assert L.hstu_time_bucket_thresholds(257, None) == 1
    # empty batches are a no-op that succeeds without touching the device
    st = L.hstu_attn_fwd(ctypes.byref(good), ctypes.byref(ok_jag), None, None, None, None, None,
                         None, None, 0, None)
    assert st == 0


def test_workspace_sizes(H):
    cfg = _cfg(H)
    a = H.layer_workspace_bytes(cfg, 1000)
    b = H.layer_workspace_bytes(cfg, 2000)
    assert 0 < a < b
    # Z (n1 bf16) + AV (H*dv bf16) + LN partials (H*2 fp32) per token
    assert a >= 1000 * (1024 * 2 + 256 * 2 + 4 * 2 * 4)
    assert H.forward_workspace_bytes(cfg, 2, 1000) > a
    assert H.lib().hstu_layer_workspace_bytes(None, 10) == 0


def test_status_strings(H):
    L = H.lib()
    for code in range(7):
        assert L.hstu_status_string(code)
    assert b"unknown" in L.hstu_status_string(99)


def test_backward_and_flag_validation_without_device(H):
    """hstu_attn_bwd / hstu_layer_bwd / cfg.flags reject bad arguments on the
    host (before any device work)."""
    L = H.lib()
    ok_jag = H.JaggedT(0, 0, 0, None, None)
    # unknown flag bits
    bad_flags = _cfg(H).c()
    bad_flags.flags = 6
    st = L.hstu_attn_fwd(ctypes.byref(bad_flags), ctypes.byref(ok_jag), None, None, None, None,
                         None, None, None, 0, None)
    assert st == 1
    # the backward has no softmax, fp32 or generalised-mask form
    soft = _cfg(H, phi2="softmax", dtype="fp16").c()
    st = L.hstu_attn_bwd(ctypes.byref(soft), ctypes.byref(ok_jag), *([None] * 12))
    assert st == 2
    f32 = _cfg(H, dtype="fp32").c()
    st = L.hstu_attn_bwd(ctypes.byref(f32), ctypes.byref(ok_jag), *([None] * 12))
    assert st == 2
    seg_jag = H.JaggedT(0, 0, 0, None, None, 16, 0)  # segments given
    good16 = _cfg(H, dtype="fp16").c()
    st = L.hstu_attn_bwd(ctypes.byref(good16), ctypes.byref(seg_jag), *([None] * 12))
    assert st == 2
    # NULL tables
    st = L.hstu_attn_bwd(ctypes.byref(good16), ctypes.byref(ok_jag), *([None] * 12))
    assert st == 1
    # layer backward: bf16 only, NULL weights / gradients rejected
    bf = _cfg(H).c()
    st = L.hstu_layer_bwd(ctypes.byref(bf), None, ctypes.byref(ok_jag), *([None] * 6), 0, None)
    assert st == 1
    assert L.hstu_layer_bwd_workspace_bytes(ctypes.byref(f32), 100) == 0
    assert L.hstu_layer_bwd_workspace_bytes(ctypes.byref(bf), 1000) > H.layer_workspace_bytes(
        _cfg(H), 1000)
