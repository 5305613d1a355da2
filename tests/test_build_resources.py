"""Every kernel of the library builds without register spills, and every
prefill kernel instance with exactly the register count its in-kernel
register split (setmaxnreg) assumes -- the host refuses to launch it
otherwise. Read from ptxas's report of the library build (CPU only)."""
import os
import re

from mqa_attention_attn_b200 import build


def _report() -> str:
    info = os.path.join(build.CSRC, "ptxas_info.txt")
    stale = (not os.path.exists(info) or not os.path.exists(build.LIB)
             or os.path.getmtime(info) < os.path.getmtime(build.LIB))
    build.build_library(force=stale)   # otherwise rebuilt only if a source changed
    return open(info).read()


def _kernels(text: str) -> dict:
    out = {}
    blocks = re.split(r"ptxas info\s+: Compiling entry function '", text)[1:]
    for blk in blocks:
        name = blk.split("'", 1)[0]
        spill = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", blk)
        regs = re.search(r"Used (\d+) registers", blk)
        assert spill and regs, name
        out[name] = (int(regs.group(1)), int(spill.group(1)), int(spill.group(2)))
    return out


def test_no_spills_and_prefill_register_count():
    ks = _kernels(_report())
    launch_regs = int(re.search(r"constexpr int kLaunchRegs = (\d+);",
                                open(os.path.join(build.CSRC, "prefill.cuh")).read()).group(1))
    prefill = {n: v for n, v in ks.items() if "prefill_kernel" in n}
    # d in {32, 64, 128} x five modes, and the FP8 mode at d = 128
    assert len(prefill) == 16, sorted(prefill)
    assert any("mla_decode_kernel" in n for n in ks)
    assert sum("decode_split_kernel" in n for n in ks) >= 15
    for name, (regs, st, ld) in ks.items():
        assert st == 0 and ld == 0, f"{name}: {st} bytes spilled, {ld} reloaded"
    for name, (regs, _, _) in prefill.items():
        assert regs == launch_regs, f"{name}: {regs} registers, the register split assumes {launch_regs}"
