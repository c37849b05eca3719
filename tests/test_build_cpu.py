"""Build properties of the hot kernels, read from the compiler's resource
report (nvcc -Xptxas -v; no GPU needed): register budgets that keep the
measured occupancy, and no spills where the kernels are bandwidth-bound.

A kernel that silently grows past its budget keeps its results but loses
its occupancy: 256-thread combine CTAs above 128 registers run one CTA per
SM instead of two (a build whose launch bounds let the per-rank combine take
152 registers measured 86.0 us against 66.6 us at 4096 tokens)."""
import os
import re
import shutil
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from combine_ep_get_10_b200 import build as BUILD  # noqa: E402

CSRC = os.path.join(ROOT, "combine_ep_get_10_b200", "csrc")


def _report(source):
    """{mangled kernel name: (registers, spill store bytes)} of one source."""
    if shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"):
        pytest.skip("nvcc not available")
    flags = [f for f in BUILD.NVCC_FLAGS if f != "--shared"]
    with tempfile.TemporaryDirectory() as tmp:
        r = subprocess.run([BUILD.nvcc()] + BUILD.ARCH_FLAGS + flags +
                           ["-I", BUILD.INCLUDE, "-I", CSRC, "-c", "-o", os.path.join(tmp, "k.o"),
                            os.path.join(CSRC, source), "-Xptxas", "-v"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    kernels, name = {}, None
    spill = 0
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            name, spill = m.group(1), 0
            continue
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and name:
            spill = int(m.group(1))
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and name:
            kernels[name] = (int(m.group(1)), spill)
            name = None
    assert kernels, r.stderr[-2000:]
    return kernels


def _pick(kernels, pattern):
    got = {k: v for k, v in kernels.items() if re.search(pattern, k)}
    assert got, "no kernel matches %r" % pattern
    return got


def test_combine_kernels_fit_two_ctas_per_sm():
    k = _report("ep_combine.cu")
    # token choice, per rank and peer rows (both output types); expert choice
    for name, (regs, _) in {**_pick(k, r"combine_kernelILi[0-3]E"), **_pick(k, r"ec_combine_kernel")}.items():
        assert regs <= 128, "%s: %d registers > 128 (two 256-thread CTAs per SM)" % (name, regs)
    # the headline combine (token choice, bf16 out) and the per-rank one do not spill
    for name, (_, spill) in {**_pick(k, r"combine_kernelILi0ELb0E"), **_pick(k, r"combine_kernelILi2ELb0E")}.items():
        assert spill == 0, "%s spills %d bytes" % (name, spill)


def test_dispatch_kernels_do_not_spill():
    k = _report("ep_dispatch.cu")
    for name, (regs, spill) in _pick(k, r"bulk_dispatch_kernelILi[0-3]E").items():
        assert spill == 0, "%s spills %d bytes" % (name, spill)
    for name, (regs, spill) in _pick(k, r"quant_dispatch_kernelILi[0-7]ELb[01]E").items():
        assert spill == 0, "%s spills %d bytes" % (name, spill)
        assert regs <= 64, "%s: %d registers > 64 (fewer than four 256-thread CTAs per SM)" % (name, regs)


def test_layout_kernels_do_not_spill():
    k = _report("ep_layout.cu")
    for pattern in (r"tc_layout_cluster_kernel", r"tc_layout_grid_kernel", r"ec_layout_cluster_kernel",
                    r"ec_(count|scan|fill|sort)_kernel"):
        for name, (_, spill) in _pick(k, pattern).items():
            assert spill == 0, "%s spills %d bytes" % (name, spill)
