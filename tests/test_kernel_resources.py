"""Register and spill budgets of the hot kernels, from ptxas (no GPU needed).

The kernels' residency rests on these numbers:

* the 4-row integer decode kernel for 2- and 4-bit codes runs 5 CTAs of 128
  threads per SM (the fifth stages its first tiles while tensor memory holds
  the other four), so it must stay at or below 96 registers (5 x 128 x 96 =
  61,440 of the SM's 65,536);
* the quantiser runs 3 CTAs of 256 threads per SM: at most 80 registers;
* no decode or prefill kernel may spill (a spill inside the per-tile loop
  costs local-memory traffic on every tile).

The test compiles the decode and append translation units with the build's
own flags plus ``-Xptxas -v`` into a temporary directory; the in-tree
library is not touched.
"""
import os
import re
import shutil
import subprocess

import pytest

from quantized_paged_kv_tq_b200 import build as B


def _ptxas(src, tmp_path):
    try:
        nvcc = B.nvcc()
    except RuntimeError:
        pytest.skip("nvcc not available")
    obj = os.path.join(str(tmp_path), os.path.splitext(src)[0] + ".o")
    cmd = [nvcc, *B.ARCH, *B.COMMON, *B.PER_FILE.get(src, []), "-Xptxas", "-v", "-c",
           os.path.join(B.CSRC, src), "-o", obj]
    out = subprocess.run(cmd, capture_output=True, text=True, check=True)
    kernels = {}
    cur = None
    for line in out.stderr.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
            kernels[cur] = {}
            continue
        if cur is None:
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            kernels[cur]["spill"] = int(m.group(1)) + int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            kernels[cur]["regs"] = int(m.group(1))
    filt = shutil.which("c++filt")
    if filt:
        names = subprocess.run([filt], input="\n".join(kernels), capture_output=True,
                               text=True).stdout.splitlines()
        kernels = {n: v for n, v in zip(names, kernels.values())}
    return kernels


def _short(name):
    """'void tq::(anonymous namespace)::k_x<4, 4>(tq::...)' -> 'k_x<4, 4>'"""
    name = name.replace("(anonymous namespace)::", "").split("(")[0]
    return name.split(" ")[-1].split("::")[-1] if "<" not in name else \
        re.sub(r"^.*?(\w+<)", r"\1", name)


def test_decode_kernels_budget(tmp_path):
    ks = _ptxas("decode_tc.cu", tmp_path)
    ks.update(_ptxas("decode.cu", tmp_path))
    short = {_short(n): v for n, v in ks.items()}
    assert any(n.startswith("k_decode_i8<4, 4>") for n in short), sorted(short)
    for name, v in short.items():
        if name.startswith(("k_decode", "k_prefill_tc")):
            assert v.get("spill", 0) == 0, (name, v)
        if name.startswith(("k_decode_i8<4, 4>", "k_decode_i8<2, 4>")):
            assert v["regs"] <= 96, (name, v)


def test_quantiser_budget(tmp_path):
    short = {_short(n): v for n, v in _ptxas("append.cu", tmp_path).items()}
    qa = {n: v for n, v in short.items() if n.startswith("k_quantize_append")}
    assert len(qa) == 5, sorted(short)          # turbo2/3/4/8 and fp8
    for name, v in qa.items():
        assert v["regs"] <= 80, (name, v)
        assert v.get("spill", 0) <= 24, (name, v)   # a few bytes outside the pass loop
