"""The product path has no fallback and no route to the oracle.

Without libfg8.so every entry point raises instead of computing anything;
the package (Python binding and CUDA sources) never imports, loads or names
the CPU oracle, which is test infrastructure only.
"""
import ast
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "fine_grained_fp8_act_b200")


def test_missing_library_raises(monkeypatch):
    import fine_grained_fp8_act_b200 as fg8
    from fine_grained_fp8_act_b200 import _capi
    monkeypatch.setattr(_capi, "_LIB_PATH", os.path.join(ROOT, "no_such_dir", "libfg8.so"))
    monkeypatch.setattr(_capi, "_lib", None)
    with pytest.raises(ImportError, match="missing"):
        fg8.fg8_version()
    with pytest.raises(ImportError):
        fg8.fg8_linear_workspace_bytes(16, 256, 256, fg8.FG8_SCALE_FLOAT)
    with pytest.raises(ImportError):
        fg8.fg8_quantize_act(0, 16, 256, 256, 0, 0, 0, None)


def test_package_sources_never_name_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for name in files:
            path = os.path.join(dirpath, name)
            if name.endswith(".py"):
                tree = ast.parse(open(path).read(), path)
                for node in ast.walk(tree):
                    mods = []
                    if isinstance(node, ast.Import):
                        mods = [a.name for a in node.names]
                    elif isinstance(node, ast.ImportFrom):
                        mods = [node.module or ""]
                    assert not any(m.split(".")[0] == "oracle" for m in mods), (path, mods)
                assert "liboracle" not in open(path).read(), path
            elif name.endswith((".cu", ".cuh", ".h")):
                text = open(path).read()
                assert "oracle" not in text.lower(), path


def test_importing_the_package_loads_no_oracle():
    code = ("import sys; import fine_grained_fp8_act_b200 as fg8; fg8.lib(); "
            "assert 'oracle' not in sys.modules, 'oracle imported'; "
            "maps = open('/proc/self/maps').read(); assert 'liboracle' not in maps, 'liboracle loaded'; "
            "assert 'libfg8.so' in maps; print('ok')")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr[-2000:]
