"""Register and spill budget of the hot kernels, from ptxas's resource report (no GPU needed).

Each bound is the occupancy the kernel is designed for: the split-role kernel's 18 warps (16
compute, 2 control; up to five per SM sub-partition) fit at <= 96 registers; two 512-thread decode blocks per SM need <= 64; the speculative kernels' 128-thread
blocks keep >= 7 per SM at <= 72. No hot kernel may spill."""
import concurrent.futures as cf
import os
import re
import subprocess

import pytest

from gated_delta_rule_62_b200 import build as B

# (source, mangled-name fragment, max registers)
BUDGET = [
    ("kda_chunk_split.cu", "split_kernelILb0E", 96),
    ("kda_chunk_split.cu", "split_kernelILb1E", 96),
    ("kda_chunk_split.cu@-DKDA_TC_INVERSE", "split_kernelILb0E", 96),  # the build option
    ("kda_chunk.cu", "chunk_kernelILi128ELb0E", 255),
    ("kda_chunk.cu", "chunk_kernelILi64ELb0E", 255),
    ("kda_chunk.cu", "chunk_kernelILi128ELb1E", 255),
    ("kda_context.cu", "seg_fixup_kernel", 255),
    ("kda_context.cu", "seg_scan_kernel", 255),
    ("kda_decode.cu", "decode_kernelI13__nv_bfloat16Li128ELi128E", 64),
    ("kda_decode.cu", "spec_kernelI13__nv_bfloat16Li128ELi128ELb0ELb1E", 72),
    ("kda_decode.cu", "spec_kernelI13__nv_bfloat16Li128ELi128ELb1ELb0E", 72),
    ("kda_decode.cu", "spec_kernelI13__nv_bfloat16Li128ELi128ELb1ELb1E", 72),
]


def _ptxas_report(spec, tmp):
    src, *defs = spec.split("@")  # source, then any -D flags of a build option
    obj = os.path.join(tmp, spec.replace("@", "_").replace("-", "") + ".o")
    cmd = [B.nvcc(), *B.ARCH, *B.NVCC_FLAGS, *defs, "-Xptxas", "-v", "-c", os.path.join(B.CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    props, name = {}, None
    for line in r.stderr.splitlines():
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            name = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and name:
            props.setdefault(name, {})["spill"] = int(m.group(1)) + int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m and name:
            props.setdefault(name, {})["regs"] = int(m.group(1))
    return props


@pytest.fixture(scope="module")
def reports(tmp_path_factory):
    tmp = str(tmp_path_factory.mktemp("ptxas"))
    srcs = sorted({s for s, _, _ in BUDGET})
    with cf.ThreadPoolExecutor(max_workers=len(srcs)) as ex:
        return dict(zip(srcs, ex.map(lambda s: _ptxas_report(s, tmp), srcs)))


@pytest.mark.parametrize("src,frag,max_regs", BUDGET, ids=[f for _, f, _ in BUDGET])
def test_hot_kernel_fits_its_register_budget(reports, src, frag, max_regs):
    hits = {n: p for n, p in reports[src].items() if frag in n}
    assert hits, f"no kernel matching {frag} in {src}"
    for name, p in hits.items():
        assert p.get("spill", 0) == 0, (name, p)
        assert p["regs"] <= max_regs, (name, p)
