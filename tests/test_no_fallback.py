"""The binding fails loudly, with no CPU or Python fallback, when the CUDA
library is missing (a copy of the package without libmoe.so is imported in a
child process)."""
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_import_without_the_library_raises(tmp_path):
    pkg = tmp_path / "group_limited_routed_moe_b200"
    shutil.copytree(os.path.join(ROOT, "group_limited_routed_moe_b200"), pkg,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc"))
    assert not any(p.suffix == ".so" for p in pkg.iterdir())
    code = ("import sys; sys.path.insert(0, sys.argv[1])\n"
            "try:\n"
            "    from group_limited_routed_moe_b200 import moe\n"
            "except ImportError as e:\n"
            "    print('IMPORT_ERROR', e); sys.exit(3)\n"
            "print('LOADED'); sys.exit(0)\n")
    r = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 3, r.stdout + r.stderr
    assert "no CPU or Python fallback" in r.stdout
