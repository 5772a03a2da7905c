"""The device-side failure path on a B200, with no GPU fault.

The library built with SOL_FAULT_TEST (libsol_fault.so) can withhold one
"P ready" arrive in every attention CTA (sol_debug_drop_arrive), a flag that
nothing else sets.  The MMA warp's bounded wait for it must run out: the
launch stops issuing, drains its copies and MMAs, frees its tensor memory,
writes no output and reports SOL_ERR_TIMEOUT through the device status
word.  The same process then runs the pass again without the drop and must
get the output of the run before the fault, bit for bit: the context stays
usable.  The fault-test library runs in a child process, so the product
library of the other tests is never replaced in this one.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, time
import numpy as np, torch
from block_sparse_video_sol_b200 import sol, synth

w = synth.tiny()
q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in synth.generate(w))
res = {}
for case, kw in [("threshold", {}), ("topk", dict(topk_ratio=0.25))]:
    p = sol.make_params(w.B, w.N, w.H, w.D, tau=w.tau, **kw)
    buf = sol.alloc_buffers(p, q.device)
    sol.forward(p, q, k, v, buf)
    res[case + "_before"] = sol.lib.sol_status_string(sol.lib.sol_last_device_status(None)).decode()
    o_before = buf.o.clone()

    sol.sol_debug_drop_arrive(0)
    buf.o.fill_(float("nan"))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    sol.forward(p, q, k, v, buf)
    st = sol.lib.sol_last_device_status(None)
    res[case + "_fault_seconds"] = time.perf_counter() - t0
    res[case + "_fault_status"] = sol.lib.sol_status_string(st).decode()
    res[case + "_fault_output_untouched"] = bool(torch.isnan(buf.o.float()).all().item())

    sol.sol_debug_drop_arrive(-1)
    sol.forward(p, q, k, v, buf)
    res[case + "_after"] = sol.lib.sol_status_string(sol.lib.sol_last_device_status(None)).decode()
    res[case + "_identical"] = bool(torch.equal(buf.o, o_before))
print(json.dumps(res))
"""


@pytest.mark.gpu
def test_withheld_arrive_times_out_and_the_context_recovers():
    from block_sparse_video_sol_b200 import build
    path = build.build(fault_test=True)
    env = dict(os.environ, SOL_LIB_PATH=path)
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-4000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    for case in ("threshold", "topk"):
        assert res[case + "_before"] == "SOL_OK", res
        assert res[case + "_fault_status"] == "SOL_ERR_TIMEOUT", res
        assert res[case + "_fault_output_untouched"], res
        assert res[case + "_fault_seconds"] < 60, res
        assert res[case + "_after"] == "SOL_OK", res
        assert res[case + "_identical"], res
