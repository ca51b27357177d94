"""The no-allocation layer entry point against the regular one.

hstu_layer_fwd_static serves callers that are given only their input and
output buffers (for example a plugin inside an engine that owns all device
memory) or that must not call cudaMalloc on a latency-critical path.  Its
scratch is a fixed array inside the library.  Two calls in a row, on two
different batches, must match hstu_layer_fwd with a caller workspace within
the parity tolerance used by the other tests; a batch too large for the
array must be refused before any launch.  This file is collected last."""
import ctypes

import numpy as np
import pytest
import torch

from gen import make_case
from hstu_testutil import assert_close, binding, config_of, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    return binding()


@pytest.mark.parametrize("seed,lengths", [(301, [37, 300, 129, 512]), (302, [1, 256, 700])])
def test_static_scratch_matches_workspace_entry(H, seed, lengths):
    for call in range(2):  # two calls in a row share the library's scratch array
        case = make_case("small-bf16", seed=seed + call, lengths=lengths, num_layers=1)
        t, jag, weights = upload(H, case)
        cfg = config_of(H, case.cfg)
        want = H.layer_fwd(cfg, weights[0], jag, t["x"]).cpu().numpy()
        got = H.layer_fwd_static(cfg, weights[0], jag, t["x"]).cpu().numpy()
        assert H.device_status() == 0
        assert_close(got, want, f"static scratch, call {call}")


def test_static_scratch_refuses_oversized_batch(H):
    cfg = H.LayerConfig(d_model=512, num_heads=8, num_pos_buckets=4096, num_time_buckets=128)
    T = 100_000  # needs far more than the fixed scratch
    need = H.layer_workspace_bytes(cfg, T)
    assert need > H.STATIC_SCRATCH_BYTES
    jag = H.JaggedT(1, T, 16384, 16, 16)  # host-side refusal: no pointer is dereferenced
    c = cfg.c()
    w = H.LayerWeightsT(16, 16, 16, 16, 16, 16, None, None)
    st = H.lib().hstu_layer_fwd_static(ctypes.byref(c), ctypes.byref(w), ctypes.byref(jag),
                                       None, None, None, None, None, None)
    assert st == 4  # HSTU_ERR_WORKSPACE_TOO_SMALL
