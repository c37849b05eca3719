"""The CPU oracle under AddressSanitizer and UndefinedBehaviorSanitizer: a
copy of ep_oracle.c is compiled with both into a temporary directory and a
subprocess (with the sanitizer runtimes preloaded) runs every oracle entry
point on sampled workloads and on the edge cases the GPU parity tests use
(empty batches, K > 32, duplicate / -1 / out-of-range ids, padded
overflow, every quantised format).  Any out-of-bounds access or undefined
operation aborts the subprocess.  The committed oracle build is untouched."""
import os
import subprocess
import sys
import tempfile

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(os.path.dirname(oracle.__file__), "ep_oracle.c")

SCRIPT = r"""
import sys
import numpy as np
import oracle
from combine_ep_get_10_b200 import workloads as W

oracle.use(oracle.load(sys.argv[1]))
r = np.random.Generator(np.random.PCG64(3))

inp = W.make_inputs(2, T=256)
idx, x, w = inp["topk_idx"], inp["x"], inp["topk_weights"]
L = oracle.tc_layout(idx, 256, 8)
d = oracle.tc_dispatch(x, idx, 256, L)
oracle.tc_combine(d["recv"], idx, 256, L, w, out_dtype=oracle.BF16)
for q in oracle.QUANT_DTYPES:
    oracle.tc_dispatch(x, idx, 256, L, out_dtype=q)
    oracle.tc_dispatch(x, idx, 256, L, mode=oracle.PADDED, max_tokens=4, out_dtype=q)  # rows past 4 overflow
rl = oracle.rank_layout(L["is_token_in_rank"])
rd = oracle.rank_dispatch(x, idx, 256, 8, rl, w, want_src=True)
oracle.rank_combine(rd["recv"], rl, out_dtype=oracle.FP32)

for T, E, R, K, p_neg, dup, p_bad in [(0, 8, 2, 2, 0.0, False, 0.0), (1, 4, 1, 4, 0.0, False, 0.0),
                                       (45, 12, 3, 36, 0.2, True, 0.02), (300, 64, 32, 6, 0.3, False, 0.1)]:
    idx = W.random_topk(r, T, E, K, p_neg=p_neg, allow_dup=dup, p_bad=p_bad)
    x = W.to_bf16_bits(r.standard_normal((T, 40)).astype(np.float32))
    w = r.random((T, K)).astype(np.float32)
    L = oracle.tc_layout(idx, E, R)
    d = oracle.tc_dispatch(x, idx, E, L)
    oracle.tc_combine(d["recv"], idx, E, L, w, out_dtype=oracle.FP32)
    oracle.tc_dispatch(x, idx, E, L, mode=oracle.PADDED, max_tokens=2)
    rl = oracle.rank_layout(L["is_token_in_rank"])
    rd = oracle.rank_dispatch(x, idx, E, R, rl, w, want_src=True)
    oracle.rank_combine(rd["recv"], rl, out_dtype=oracle.BF16)

i4 = W.make_inputs(4, T=512)
L4 = oracle.ec_layout(i4["token_indices"], 512, 8)
y4 = oracle.ec_dispatch(i4["x"], i4["token_indices"])
oracle.ec_combine(y4, L4, i4["expert_weights"], 512, out_dtype=oracle.FP32)
for T, E, C, p_neg, p_bad in [(50, 8, 16, 0.0, 0.0), (20, 16, 8, 0.2, 0.05), (5, 40, 6, 0.1, 0.0), (1, 3, 2, 0.5, 0.0)]:
    ti = W.random_token_indices(r, T, E, C, p_neg=p_neg, p_bad=p_bad)
    L = oracle.ec_layout(ti, T, 2)
    x = W.to_bf16_bits(r.standard_normal((T, 16)).astype(np.float32))
    y = oracle.ec_dispatch(x, ti, recv=np.full((E * C, 16), 0x7FC1, np.uint16))
    oracle.ec_combine(y, L, r.standard_normal((E, C)).astype(np.float32), T, out_dtype=oracle.BF16)
print("sanitized oracle ok")
"""


def _runtime(name):
    try:
        path = subprocess.run(["gcc", "-print-file-name=" + name], capture_output=True, text=True,
                              check=True).stdout.strip()
    except (OSError, subprocess.CalledProcessError):
        return None
    return path if os.path.isabs(path) and os.path.exists(path) else None


def test_oracle_is_clean_under_asan_and_ubsan():
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if asan is None or ubsan is None:
        pytest.skip("gcc sanitizer runtimes not installed")
    with tempfile.TemporaryDirectory() as d:
        lib = os.path.join(d, "libep_oracle_san.so")
        subprocess.check_call(["gcc", "-std=c99", "-O1", "-g", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                               "-shared", "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined",
                               "-fno-omit-frame-pointer", "-o", lib, SRC, "-lm"])
        env = dict(os.environ, LD_PRELOAD=asan + ":" + ubsan, ASAN_OPTIONS="detect_leaks=0:abort_on_error=1",
                   UBSAN_OPTIONS="print_stacktrace=1:halt_on_error=1",
                   PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
        res = subprocess.run([sys.executable, "-c", SCRIPT, lib], env=env, capture_output=True, text=True,
                             timeout=600, cwd=ROOT)
    assert res.returncode == 0 and "sanitized oracle ok" in res.stdout, (res.stdout[-2000:], res.stderr[-4000:])
