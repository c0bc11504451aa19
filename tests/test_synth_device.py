"""The device twin of the generator reproduces the host generator bit for bit."""
import os

import numpy as np
import pytest
import torch

import synth
from synth import device as sdev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    assert torch.cuda.is_available()
    if not os.path.exists(sdev.LIB_PATH):
        sdev.build()


@pytest.mark.parametrize("name,kind,layer", [("tiny_f32", "K", 0), ("tiny_f32", "V", 0),
                                             ("llama1b_32k", "K", 0), ("llama1b_32k", "V", 0),
                                             ("qwen1p5b_128k", "K", 0),
                                             ("llama1b_stack16_b8_128k", "K", 9),
                                             ("llama1b_32k", "KD", 0), ("llama1b_32k", "VD", 0)])
def test_device_fill_matches_host(name, kind, layer):
    w = synth.WORKLOADS[name]
    H = {"K": w.h_k, "V": w.h_v}.get(kind, w.dense_hkv)
    cap = min(w.l_kv, 6000)
    dt = torch.float32 if w.dtype == synth.F32 else torch.int16
    t = torch.empty(w.B, H, cap, w.d, dtype=dt, device="cuda")
    sdev.fill(t, w, layer, kind)
    dev = t.cpu().numpy()
    if dt == torch.int16:
        dev = dev.view(np.uint16)
    for b in sorted({0, w.B - 1}):
        for h in sorted({0, H - 1}):
            host = synth.cache_rows(w, layer, kind, b, h, 0, cap)
            np.testing.assert_array_equal(dev[b, h].view(np.uint8), host.view(np.uint8))
