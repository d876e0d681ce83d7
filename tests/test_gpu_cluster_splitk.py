"""Cluster split-K gives the slab path's results bit for bit (the same split order).

The switch QLORA_CLUSTER_SPLITK is read once per process, so each setting runs in a child process that writes its
outputs to a file."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from qlora_fine_tuning_blockwise_b200 import inputs as I, ops
out = {}
for name in ("attn_2048x4096x4096_r16", "mlpdown_4096x11008x4096_r64"):
    w = I.WORKLOADS[name]
    d = I.make_linear_inputs(w)
    layer = ops.QLoRALinear(torch.from_numpy(d["W"]).cuda(), d["A"].cuda(), d["B"].cuda(), d["s"])
    x, dy = d["x"].cuda(), d["dy"].cuda()
    y, su = layer.forward(x)
    dx, dA, dB = layer.backward(dy, x, su=su)
    torch.cuda.synchronize()
    for k, t in (("y", y), ("su", su), ("dx", dx), ("dA", dA), ("dB", dB)):
        out[name + "/" + k] = t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).cpu().numpy()
np.savez(sys.argv[2], **out)
'''


def run(setting, path):
    env = dict(os.environ, QLORA_CLUSTER_SPLITK=setting)
    subprocess.run([sys.executable, "-c", CHILD, ROOT, path], check=True, env=env, timeout=600)
    return np.load(path)


def test_cluster_splitk_equals_slabs(tmp_path):
    a = run("1", str(tmp_path / "on.npz"))
    b = run("0", str(tmp_path / "off.npz"))
    assert set(a.files) == set(b.files)
    for k in a.files:
        assert np.array_equal(a[k], b[k]), k
