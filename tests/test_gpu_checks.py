"""The bounds-checked build (libsage_fp4_checks.so, compiled with SAGE_CHECKS) on the GPU:
the tiny, ragged, packed, grouped-head, Q-smoothing, second-level-scale and 8-bit problems
run with every computed global index checked before its access. The checks must pass
(device error word 0) and the results must still match the oracle at the parity bar. The
build's self-test switch then takes the output's extent as 0: every output store must
fail its check, be skipped (the output keeps its sentinel) and be reported as
SAGE_ERR_BOUNDS, with nothing faulting. Runs in a child process that loads the checked
library, so that the rest of the GPU suite keeps the regular one."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

CHILD = r'''
import json, sys
import numpy as np, torch
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import microscaling_fp4_quantized_b200 as sage
import oracle
from microscaling_fp4_quantized_b200 import workloads as W
assert sage.lib().sage_fp4_bounds_checked() == 1
res = {}
def dense(name, wl):
    q, k, v = W.make_inputs(wl, device="cuda")
    out = sage.attn(q, k, v, causal=wl.causal, sm_scale=wl.sm_scale)
    torch.cuda.synchronize()
    word = sage.device_error()
    f = lambda t: t.float().cpu().numpy().reshape(wl.B * wl.H, wl.N, wl.D)
    em, _ = oracle.attention(f(q), f(k), f(v), wl.causal, wl.sm_scale, Bk=128)
    m = oracle.metrics(f(out), em)
    res[name] = {"word": word, "cos": m["cos"], "max_abs_frac": m["max_abs"] / float(np.abs(f(v)).max())}
dense("tiny", W.TINY)
dense("ragged_causal_d128", W.custom(1, 2, 300, 128, causal=True, seed=71))
dense("ragged_d64", W.custom(2, 1, 200, 64, causal=False, seed=72))
dense("short_persistent", W.custom(4, 8, 384, 128, causal=False, seed=73))
def general(name, w, precision="fp4"):
    x = W.make_general_inputs(w, "cuda")
    if w.packed:
        out = sage.sageattn_varlen(x["q"], x["k"], x["v"], x["cu_seqlens_q"], x["cu_seqlens_k"], max(w.lens_q),
                                   max(w.lens_k), is_causal=w.causal, gscale=w.gscale, smooth_q=w.smooth_q,
                                   precision=precision)
    else:
        out = sage.sageattn(x["q"], x["k"], x["v"], tensor_layout=w.layout, is_causal=w.causal,
                            gscale=w.gscale, smooth_q=w.smooth_q, precision=precision)
    torch.cuda.synchronize()
    res[name] = {"word": sage.device_error(), "finite": bool(torch.isfinite(out.float()).all())}
general("packed_gqa_head_scale", W.general("g1", 4, 2, 128, (5, 0, 300, 128, 1, 400), causal=True, seed=74,
                                           gscale="head"))
general("qsmooth_tensor_scale", W.general("g2", 4, 2, 64, (130, 0, 257), seed=75, smooth_q=True, gscale="tensor"))
general("nhd_fp16_cross", W.general("g3", 2, 2, 64, (200,), (333,), packed=False, layout="NHD",
                                    dtype=torch.float16, seed=76))
general("eight_bit_packed", W.general("g4", 4, 2, 128, (5, 300, 1), seed=77), precision="8bit")
# Self-test: the output's extent taken as 0 -> every output store refused and reported.
wl = W.custom(1, 2, 256, 128, seed=78)
q, k, v = W.make_inputs(wl, device="cuda")
out = torch.full_like(q, 7.0)
sage.set_debug_flags(2)
try:
    sage.attn(q, k, v, out=out)
    torch.cuda.synchronize()
finally:
    sage.set_debug_flags(0)
res["self_test"] = {"word": sage.device_error(), "untouched": bool((out == 7.0).all())}
print(json.dumps(res))
'''


def test_bounds_checked_build(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from microscaling_fp4_quantized_b200 import build as b
    lib = b.build(checks=True)
    env = dict(os.environ, SAGE_FP4_LIB=lib)
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], capture_output=True, text=True,
                       env=env, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    print("\n" + json.dumps(res, indent=1))
    for name in ("tiny", "ragged_causal_d128", "ragged_d64", "short_persistent"):
        assert res[name]["word"] == 0, (name, res[name])
        assert res[name]["cos"] >= 0.999 and res[name]["max_abs_frac"] <= 1e-2, (name, res[name])
    for name in ("packed_gqa_head_scale", "qsmooth_tensor_scale", "nhd_fp16_cross", "eight_bit_packed"):
        assert res[name]["word"] == 0 and res[name]["finite"], (name, res[name])
    assert res["self_test"]["word"] & 4, res["self_test"]          # reported as a bounds failure
    assert res["self_test"]["untouched"], res["self_test"]          # and no store went through
