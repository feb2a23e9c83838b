"""Without the built C-ABI library the product path fails loudly: the
package's configs and synth still import, but the first use of a library name
raises ImportError (there is no CPU or library fallback)."""
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "mixture_experts_layer_36_b200"


def test_missing_library_raises_importerror(tmp_path):
    dst = tmp_path / PKG
    dst.mkdir()
    for name in os.listdir(os.path.join(ROOT, PKG)):
        if name.endswith(".py"):                 # the Python files only: no libmoe.so
            shutil.copy(os.path.join(ROOT, PKG, name), dst / name)
    code = (f"import {PKG} as m\n"
            f"from {PKG} import configs, synth\n"
            "synth.make_tokens(configs.TINY, 'cpu')\n"
            "try:\n"
            "    m.moe_capacity(64, 8, 2, 1.25)\n"
            "except ImportError as e:\n"
            "    print('ImportError:', e)\n"
            "else:\n"
            "    print('no error')\n")
    env = dict(os.environ, PYTHONPATH=str(tmp_path))
    out = subprocess.run([sys.executable, "-c", code], cwd=str(tmp_path), env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "ImportError: libmoe.so not built" in out.stdout, out.stdout
