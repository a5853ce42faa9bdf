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


def test_profile_commands_run_committed_files():
    """Every profile summary gives its command; its bench.py part names real options and workloads."""
    pdir = os.path.join(ROOT, "profiles")
    for name in sorted(os.listdir(pdir)):
        if not name.endswith(".md"):
            continue
        text = open(os.path.join(pdir, name)).read().replace("\\\n", " ")
        assert "--clock-control none" in text or "ncu" not in text, name
        cmds = re.findall(r"(python (?:bench\.py|-m [\w.]+)[^\n`]*)", text)
        assert cmds, f"{name}: no command"
        for cmd in cmds:
            argv = shlex.split(cmd)
            if argv[1] == "-m":
                assert argv[2] == "fine_grained_fp8_act_b200.build", (name, cmd)
                continue
            args = argv[2:]
            assert {a for a in args if a.startswith("--")} <= KNOWN, (name, cmd)
            if "--workload" in args:
                wl = args[args.index("--workload") + 1]
                assert wl == "moe_dsv3" or bench.workload_layers(wl), (name, cmd)
