"""The bounds-checked build (compiled with -DSAGA_CHECK, loaded when
SAGA_CHECKED_BUILD=1): on valid inputs no index check fails, so the device
error word stays 0, and the checks change no arithmetic, so every output
equals the ordinary build's bit for bit. Each build runs in its own process
(the binding loads one library per process)."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# A refresh, two plain steps, an exact top-N step and the dense step on a
# ragged batch (one empty sequence, tails shorter than a tile), both head
# dimensions; outputs, counts, thresholds and the error word to an .npz.
CHAIN = r"""
import sys
import numpy as np, torch
import synth
import sparse_decode_attention_step_b200 as saga
saga.load()
res = {}
for d, hq, hk, hv in ((64, 16, 2, 4), (128, 12, 1, 4)):
    w = synth.Workload("checked", synth.BF16, B=3, h_q=hq, h_k=hk, h_v=hv, d=d, l_kv=1300,
                       N=40, R=2, steps=3, seed=2468 + d)
    lens = np.array([1300, 0, 301], dtype=np.int32)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
    K = dev(synth.cache(w, 0, "K", hk, 1300, lens))
    V = dev(synth.cache(w, 0, "V", hv, 1300, lens))
    qs = synth.queries(w, 0, 3)
    shp = saga.shape(w.B, hq, hk, hv, d, w.dtype, 1300)
    ws = saga.Workspace(shp, w.N)
    l = torch.from_numpy(lens).cuda()
    tau = torch.zeros(w.B, hq, device="cuda")
    out = torch.zeros(w.B, hq, d, device="cuda")
    cnt = torch.zeros(w.B, hq, dtype=torch.int32, device="cuda")
    saga.refresh_threshold(shp, dev(qs[0]), K, l, w.N, tau, ws, V=V, out=out, sel_count=cnt)
    res[f"d{d}_refresh"] = out.cpu().numpy().copy()
    res[f"d{d}_tau"] = tau.cpu().numpy().copy()
    for t in (1, 2):
        saga.decode_step(shp, dev(qs[t]), K, V, l, tau, out, ws, sel_count=cnt)
        res[f"d{d}_step{t}"] = out.cpu().numpy().copy()
        res[f"d{d}_cnt{t}"] = cnt.cpu().numpy().copy()
    saga.topn_step(shp, dev(qs[2]), K, V, l, w.N, out, ws, sel_count=cnt)
    res[f"d{d}_topn"] = out.cpu().numpy().copy()
    res[f"d{d}_topn_cnt"] = cnt.cpu().numpy().copy()
    res[f"d{d}_err"] = np.array([saga.read_device_error(ws)])
np.savez(sys.argv[1], **res)
"""


def run_chain(tmp_path, checked):
    path = str(tmp_path / ("checked.npz" if checked else "plain.npz"))
    env = dict(os.environ)
    env["SAGA_CHECKED_BUILD"] = "1" if checked else "0"
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    r = subprocess.run([sys.executable, "-c", CHAIN, path], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return dict(np.load(path))


def test_checked_build_agrees_bitwise_and_reports_nothing(tmp_path):
    from sparse_decode_attention_step_b200 import build
    if not os.path.exists(build.CHECK_LIB_PATH):
        build.build(check=True)
    plain = run_chain(tmp_path, False)
    checked = run_chain(tmp_path, True)
    assert set(plain) == set(checked)
    for k in plain:
        if k.endswith("_err"):
            assert int(plain[k][0]) == 0 and int(checked[k][0]) == 0, k
        else:
            np.testing.assert_array_equal(plain[k].view(np.uint32) if plain[k].dtype == np.float32
                                          else plain[k],
                                          checked[k].view(np.uint32) if checked[k].dtype == np.float32
                                          else checked[k], err_msg=k)
