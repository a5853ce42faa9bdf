"""The README's bench.py command lines name workloads and options that exist."""
import os
import re
import shlex

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
# the options bench.py defines
KNOWN = set(re.findall(r'add_argument\("(--[a-z-]+)"', open(os.path.join(ROOT, "bench.py")).read()))


def test_readme_bench_commands_parse():
    text = open(os.path.join(ROOT, "README.md")).read()
    cmds = [ln.split("#")[0].strip() for ln in text.splitlines() if re.match(r"\s*python bench\.py", ln)]
    assert len(cmds) >= 5
    for cmd in cmds:
        argv = shlex.split(cmd)[2:]
        wl = argv[argv.index("--workload") + 1] if "--workload" in argv else "esm2_ffn"
        if wl != "moe_dsv3":
            assert bench.workload_layers(wl), cmd
        opts = {a for a in argv if a.startswith("--")}
        assert opts <= KNOWN, (cmd, opts - KNOWN)
