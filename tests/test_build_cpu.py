"""Register and spill budgets of the hot kernels, read from the ptxas report
the build saves for every source (nvcc -Xptxas -v, sm_100a).  These are the
figures the kernels' performance depends on: the tensor-core GEMMs keep every
value in registers, and the activation quantiser's two builds stay within the
registers that give them 2048 (wide) and 1536 (deep) resident threads."""
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BUILD = os.path.join(ROOT, "binary_weight_transformer_b200", "_build")


@pytest.fixture(scope="module")
def kernels():
    from binary_weight_transformer_b200 import _build
    _build.build()
    found = []
    for path in glob.glob(os.path.join(BUILD, "*.ptxas.txt")):
        text = open(path).read()
        for m in re.finditer(r"Compiling entry function '([^']+)'.*?(\d+) bytes spill stores.*?Used (\d+) registers",
                             text, re.S):
            found.append((m.group(1), int(m.group(2)), int(m.group(3))))
    if not found:
        pytest.skip("no ptxas report (library built elsewhere)")
    return found


@pytest.mark.parametrize("kernel", ["gemm_kernel", "gemm_splitk_kernel", "gemm_pair_kernel", "gemm_ts_kernel",
                                    "gemm_ts_pair_kernel", "skinny_mma_kernel"])
def test_tensor_core_kernels_do_not_spill(kernels, kernel):
    pat = re.compile(r"\d+" + kernel + r"I")  # mangled name: <length><name>I<template args>
    hits = [(n, s) for n, s, _ in kernels if pat.search(n)]
    assert hits, kernel
    assert all(s == 0 for _, s in hits), [h for h in hits if h[1]]


def test_act_quant_builds_fit_their_occupancy(kernels):
    # act_quant_regs<T, TPR, VPT, SM_THREADS>: mangled as ...act_quant_regsI<T>Li<TPR>ELi<VPT>ELi<SM>E...
    pat = re.compile(r"act_quant_regsI\w+?Li(\d+)ELi(\d+)ELi(\d+)E")
    seen = 0
    for name, _, regs in kernels:
        m = pat.search(name)
        if not m:
            continue
        tpr, vpt, sm_threads = map(int, m.groups())
        block = max(tpr, 256)
        if sm_threads // block >= 1 and block * (sm_threads // block) == sm_threads:
            assert regs * sm_threads <= 65536, (name, regs)
        seen += 1
    assert seen >= 28
