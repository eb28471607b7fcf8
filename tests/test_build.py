"""Build-time checks of libsala (CPU only): the register count ptxas gave
the kernels whose warp roles reallocate registers with setmaxnreg, read from
the `ptxas -v` report the build writes beside the library."""
import json
import os

import pytest

from hybrid_sparse_linear_lightning_b200 import build as B


def test_parse_ptxas_report_lines():
    text = ("ptxas info    : Compiling entry function '_ZN4sala20linear_segout_kernelEv' for 'sm_100a'\n"
            "ptxas info    : Function properties for _ZN4sala20linear_segout_kernelEv\n"
            "    0 bytes stack frame, 0 bytes spill stores, 0 bytes spill loads\n"
            "ptxas info    : Used 128 registers, used 1 barriers, 1024 bytes cmem[0]\n"
            "ptxas info    : Compiling entry function '_Z3fooPf' for 'sm_100a'\n"
            "ptxas info    : Used 40 registers, used 0 barriers\n")
    regs = B.parse_ptxas(text)
    assert regs == {"_ZN4sala20linear_segout_kernelEv": 128, "_Z3fooPf": 40}
    B.check_register_splits(regs)
    with pytest.raises(RuntimeError):
        B.check_register_splits({"_ZN4sala20linear_segout_kernelEv": 96})


def test_built_library_register_split():
    if not os.path.exists(B.REPORT):
        pytest.skip("library not built by build.py in this tree")
    with open(B.REPORT) as f:
        regs = json.load(f)["registers_per_thread"]
    seg = [v for k, v in regs.items() if "linear_segout_kernel" in k]
    assert seg and all(v == B.REGISTER_SPLIT_KERNELS["linear_segout_kernel"] for v in seg)
