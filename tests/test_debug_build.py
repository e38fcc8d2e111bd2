"""The bounds-checked debug build (libqlora_debug.so, -DQLORA_DEBUG), host side: it builds, exports
every symbol the header declares, says what it is, and the binding loads it when the environment
sets QLORA_LIBRARY=debug (the default build otherwise)."""
import ctypes
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "qlora.h")).read()
    return sorted(set(re.findall(r"QLORA_API\s+[\w\s\*]+?\b(qlora_\w+)\s*\(", src)))


def test_debug_library_exports_every_symbol():
    from bit_quantized_base_b200 import build
    path = build.build(debug=True)
    assert path.endswith("libqlora_debug.so")
    L = ctypes.CDLL(path)
    for n in _declared():
        getattr(L, n)
    L.qlora_build_info.restype = ctypes.c_char_p
    assert b"debug" in L.qlora_build_info()
    R = ctypes.CDLL(build.build())
    R.qlora_build_info.restype = ctypes.c_char_p
    assert b"debug" not in R.qlora_build_info()


def test_binding_selects_the_debug_build_from_the_environment():
    from bit_quantized_base_b200 import build
    build.build()
    build.build(debug=True)
    code = ("from bit_quantized_base_b200 import qlora as Q; import os; "
            "print(os.path.basename(Q.LIB_PATH), Q.lib.qlora_build_info().decode())")
    for env_value, lib, tag in (("debug", "libqlora_debug.so", "debug"), ("", "libqlora.so", None)):
        env = dict(os.environ, QLORA_LIBRARY=env_value, PYTHONPATH=ROOT)
        out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                             text=True, timeout=300)
        assert out.returncode == 0, out.stderr
        name, info = out.stdout.strip().split(" ", 1)
        assert name == lib
        assert (tag in info) if tag else ("debug" not in info)
