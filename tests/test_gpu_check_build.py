"""The checking build (libmuir_check.so, compiled with -DMUIR_CHECK): the same
kernels with device-side index checks in the central access helpers (shared-memory
stores and bulk-copy destinations against the CTA's shared-memory window, token,
batch and head indices of the input tensors, Gram image rows and columns). A
failed check is recorded in the status word, which muir_device_status() reports
as MUIR_ERR_BOUNDS; nothing traps. Each case runs in a child process that loads
the checking build through the package's own binding (MUIR_LIBRARY), on the tiny
fp32 workload and a bf16 case, and compares with the fp64 oracle."""
import os
import subprocess
import sys

import pytest

from gated_delta_rule_muir_b200 import _native as N

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200 import _native as N
from gated_delta_rule_muir_b200.inputs import make_inputs
from oracle import muir_oracle as orc
from tests.gpu_util import INPUT_NAMES, to_dev, rel_err
assert N.LIB_PATH.endswith("libmuir_check.so"), N.LIB_PATH
B, T, H, dk, dv, chunk, dtype = [int(x) if x.isdigit() else x for x in sys.argv[2:9]]
d = make_inputs(B, T, H, dk, dv, dtype=dtype, seed=0, with_state=True, with_grads=True)
t = to_dev(d, dtype)
a = [t[n] for n in INPUT_NAMES]
y, S = muir.chunk_fwd(*a, chunk=chunk, S0=t["S0"])
gr = muir.chunk_bwd(*a, t["dy"], chunk=chunk, S0=t["S0"], dS_T=t["dS_T"])
Sd = t["S0"].clone()
yd = muir.decode_step(Sd, *[x[:, 0].contiguous() for x in a[:8]], t["r"])
torch.cuda.synchronize()
status = muir.device_status()
o = [d[n] for n in INPUT_NAMES]
y_ref, S_ref = orc.forward(*o, S0=d["S0"])
g_ref = orc.backward(*o, d["dy"], S0=d["S0"], dS_T=d["dS_T"])
ty, tg = (1e-4, 1e-3) if dtype == "f32" else (2e-2, 5e-3)
errs = [rel_err(y, y_ref), rel_err(S, S_ref)] + [rel_err(gr[n], g_ref[n]) for n in ("dq", "dk", "dv", "de", "dw", "dg", "dlog_alpha")]
print("status", status, N.load().muir_last_error().decode(), "errors", ["%.2e" % e for e in errs])
assert status == 0, status
assert errs[0] < ty and errs[1] < (1e-4 if dtype == "f32" else 1e-3), errs
assert max(errs[2:]) < tg, errs
print("CHECK_BUILD_OK")
'''


@pytest.mark.parametrize("case", [("1", "256", "2", "32", "32", "64", "f32"),
                                  ("1", "384", "2", "128", "64", "128", "bf16"),
                                  ("1", "512", "1", "64", "128", "256", "f32")])
def test_checking_build_runs_clean(cuda_ok, case):
    assert os.path.exists(N.CHECK_LIB_PATH), "libmuir_check.so is built by __graft_entry__.build()"
    env = dict(os.environ, MUIR_LIBRARY=N.CHECK_LIB_PATH)
    res = subprocess.run([sys.executable, "-c", CHILD, ROOT, *case], env=env, capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0 and "CHECK_BUILD_OK" in res.stdout, res.stdout[-3000:] + res.stderr[-3000:]
