"""The bounds-guarded debug build (libbbc_debug.so) on the GPU.

Every global access whose address a kernel computes is checked there against its buffer's
extent; a failed check skips the access and sets a bit that bbc_debug_status reports. The script
below runs in a child process with BBC_LIBRARY pointing at the debug build: every operation of
the library on ragged and aligned sizes (all K, dtypes, E4M4, nested fused and chained, nested
quantize with a two-level tree, both fused linear paths), each compared bit for bit with the
oracle (the linear layers within their derived bound), and then asserts that no guard fired.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import numpy as np, torch
import blockwise_bit_codebook_b200 as bbc
import oracle
from blockwise_bit_codebook_b200 import synthetic
from tests import test_gpu_kbit as tk, test_gpu_e4m4 as te, test_gpu_nested as tn
from tests import test_gpu_nested_quant as tq, test_gpu_linear as tl
assert bbc.bbc_is_debug_build(), bbc.library_path()
bbc.bbc_debug_status(reset=True)
dts = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}
cases = 0
# k-bit quantize / dequantize (fp32 and E4M4 absmax): ragged, aligned, whole-block and half-block forms
for K in (2, 3, 4, 5):
    cb = oracle.normal_float_codebook(K)
    for name, dt in dts.items():
        for n in (1, 31, 33, 4096 + 37, 32 * 1024 * 9 + 5, 32 * 8192):
            x = synthetic.weights(n, std=0.02, seed=n + K, dtype=dt)
            p, a = tk.check_quantize(bbc, x, K, cb, what="debug")
            tk.check_dequantize(bbc, p, a, cb, K, n, name, what="debug")
            te.roundtrip(bbc, x, K, what="debug")
            cases += 3
# nested dequant (fused; NF4 and FP4) and the three-launch chain
for bs in (32, 64, 256, 4096):
    for n in (bs * 300 + 37, bs * 256 * 3):
        for name in ("bf16", "f32"):
            for fmt in ("nf4", "fp4"):
                y = tn.run_both(bbc, n, bs, name, fmt, seed=bs)
                codes, q, a2, off = synthetic.nested_state(n, bs, seed=bs)
                code2, code4 = tn.tables(fmt)
                yc = bbc.dequantize_4bit_nested_chain(codes.cuda(), q.cuda(), torch.from_numpy(code2).cuda(),
                                                      a2.cuda(), float(off), torch.from_numpy(code4).cuda(),
                                                      n, bs, dts[name])
                torch.cuda.synchronize()
                assert torch.equal(yc[:n].view(torch.uint8), y[:n].view(torch.uint8)), (bs, n, name, fmt)
                cases += 2
# 4-bit and nested quantize: one tree level and two (4,198,405 outer blocks of 32)
for bs in (32, 64, 1024):
    tq.check_q4(bbc, synthetic.weights(bs * 500 + 17, std=0.02, seed=bs, dtype=torch.bfloat16), bs, tq.NF4, what="debug")
    cases += 1
tq.check_nested(bbc, synthetic.weights(64 * 256 * 7 + 37, std=0.02, seed=9, dtype=torch.bfloat16), 64, what="debug")
tq.check_nested(bbc, synthetic.weights(32 * (2048 * 2048 + 2048 * 2 + 5) - 7, std=0.02, seed=77,
                                       dtype=torch.bfloat16), 32, what="debug two levels")
cases += 2
# fused linear: warp-level MMA (M <= 32) and tcgen05 (M > 32) paths, nested and k-bit weights
for M in (1, 9, 32, 64, 256):
    tl.run_case(bbc, M, 256, 1024, 64, "bf16", seed=M)
    tl.run_kbit_case(bbc, M, 256, 1024, 4, "bf16", seed=M)
    cases += 2
torch.cuda.synchronize()
status = bbc.bbc_debug_status(reset=True)
assert status == 0, f"bounds guards fired: {status:#x}"
assert bbc.bbc_wait_timeouts() == 0
print("debug build: %d cases, guard status 0" % cases)
'''


def test_debug_build_runs_every_operation_with_no_guard_firing():
    from blockwise_bit_codebook_b200 import build
    lib = build.build(debug=True)
    env = dict(os.environ, BBC_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=1200)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "guard status 0" in r.stdout
