"""Build-time checks of the kernels' register use (ptxas -v, no GPU).

The attention kernel's warp roles trade registers with setmaxnreg, which only
redistributes what the CTA was launched with; the kernel must therefore be
built with exactly kLaunchRegs per thread (the host refuses to launch it with
fewer).  With the 216 / 72 split it does not spill today; the bound below
leaves a little room.  The other kernels must not spill at all."""
import os
import re

from block_sparse_prefill_b200 import build as b

ATTENTION = os.path.join(b.CSRC, "attention.cu")


def _launch_regs():
    return int(re.search(r"constexpr int kLaunchRegs = (\d+);", open(ATTENTION).read()).group(1))


def test_kernel_registers_and_spills():
    rep = b.ptxas_report()
    names = [k["name"] for k in rep]
    att = [k for k in rep if "attention_kernel" in k["name"]]
    assert len(att) == 4, names                      # bf16 and e4m3, without and with the variance term
    for k in att:
        assert k["regs"] == _launch_regs(), k
        assert k["spill_stores"] <= 16 and k["spill_loads"] <= 64, k
    for short in ("pool_kernel", "score_kernel", "meanlp_kernel", "setup_kernel"):
        ks = [k for k in rep if short in k["name"]]
        assert ks, short
        for k in ks:
            assert k["spill_stores"] == 0 and k["spill_loads"] == 0, k
            assert k["regs"] <= 255, k
