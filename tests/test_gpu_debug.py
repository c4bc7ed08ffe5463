"""The W4_DEBUG build on the GPU: the decode (M = 1 GEMV, M = 4 warp-MMA GEMV,
M = 16 tcgen05 decode on both its whole-row-block and split paths), prefill
and quantizer kernels with every bounds check compiled in, on small ragged
shapes, each checked against the oracle, and the device status word clean
(no check failed, no wait ran out).  Runs in a child process with
W4_DEBUG=1, which loads libw4a16_debug.so."""
import os
import subprocess
import sys

import pytest

from weight_only_int4_pack_b200 import build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import numpy as np, torch
import synth
import weight_only_int4_pack_b200 as w4
from helpers import check_y, oracle_linear, oracle_quantize
assert w4.w4_debug_build()
assert w4.w4_device_status(True) == w4.W4_OK
dev = "cuda"
cases = [  # (M, N, K, sym, dtype)
    (1, 1000, 4096, False, "f16"), (1, 333, 1024, True, "bf16"),
    (4, 1000, 2048, False, "f16"), (7, 129, 4096, True, "bf16"),
    (16, 4100, 4096, False, "f16"), (16, 300, 8192, True, "bf16"), (24, 2000, 6144, False, "f16"),
    (256, 1000, 4096, False, "bf16"), (200, 513, 1024, True, "f16"),
]
for (M, N, K, sym, dt) in cases:
    W = synth.weights(N, K, 0.02, 11 + M + N, outlier_frac=0.001, dtype=dt)
    p, s, z = w4.w4_quantize(W.to(dev), 128, sym=sym)
    po, so, zo = oracle_quantize(W, 128, sym)
    assert np.array_equal(p.cpu().numpy(), po), ("codes", M, N, K)
    assert np.array_equal(s.cpu().numpy(), so), ("scales", M, N, K)
    X = synth.activations(M, K, 5 + M, salient_frac=0.01, dtype=dt)
    Y = w4.w4a16_gemm(X.to(dev), p, s, None if sym else z)
    torch.cuda.synchronize()
    check_y(Y, oracle_linear(X, po, so, None if sym else zo, K), f"debug M={{M}} N={{N}} K={{K}}")
    st = w4.w4_device_status(False)
    assert st == w4.W4_OK, (M, N, K, st, w4.w4_debug_first_failure())
    print("case", M, N, K, "clean", flush=True)
# the quantizer with a folded column scale, a ragged row count
W = synth.weights(77, 2048, 0.02, 3)
cs = torch.rand(2048, dtype=torch.float32) + 0.5
p, s, z = w4.w4_quantize(W.to(dev), 128, sym=False, col_scale=cs.to(dev))
torch.cuda.synchronize()
assert w4.w4_device_status(True) == w4.W4_OK, w4.w4_debug_first_failure()
assert w4.w4_debug_first_failure() == (0, 0)
print("ok")
"""


def test_debug_build_runs_clean_against_the_oracle():
    build.build(debug=True)
    env = dict(os.environ, W4_DEBUG="1")
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=400)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-3000:] + r.stderr[-4000:]
