"""The C ABI from plain C: ``tests/abi_from_c.c`` includes
``include/xlstm_mlstm.h``, is compiled as C11 with warnings as errors, links
``libxlstm_mlstm.so`` and calls the entry points on host-only paths (version,
status strings, workspace queries, argument validation).  No device is
needed."""
import os
import shutil
import subprocess
import tempfile

from linear_rnn_mlstm_b200 import binding as xb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_header_compiles_as_c11_and_the_library_links_and_answers():
    gcc = shutil.which("gcc")
    assert gcc, "gcc is needed"
    xb.load()                                   # the library is built
    libdir = os.path.dirname(xb.LIB_PATH)
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "abi_from_c")
        cmd = [gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
               "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_from_c.c"),
               "-o", exe, "-L", libdir, "-l:libxlstm_mlstm.so", f"-Wl,-rpath,{libdir}"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
        assert r.returncode == 0, r.stdout + r.stderr
        assert r.stdout.count("ok ") == 10
