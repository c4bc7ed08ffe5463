"""The W4_DEBUG build (in-kernel bounds checks; include/w4a16.h), checked
without a GPU: it compiles for sm_100a, loads, exports every function the
header declares, reports itself as the debug build, and the normal build
does not.  Both libraries are loaded in child processes that see no GPU, so
nothing here can reach a device."""
import os
import re
import subprocess
import sys

from weight_only_int4_pack_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROBE = r"""
import os, re, sys
sys.path.insert(0, {root!r})
import weight_only_int4_pack_b200 as w4
lib = w4.load()
assert os.path.basename(w4.lib_path) == {name!r}, w4.lib_path
names = set()
for fn in os.listdir(os.path.join({root!r}, "include")):
    if fn.endswith(".h"):
        src = open(os.path.join({root!r}, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(m.group(1) for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(w4\w*)\s*\(", src, flags=re.M))
missing = [n for n in sorted(names) if not hasattr(lib, n)]
assert not missing, missing
assert w4.w4_debug_build() == {debug}, w4.w4_debug_build()
assert w4.w4_status_string(w4.W4_ERR_BOUNDS) == "W4_ERR_BOUNDS"
print("ok")
"""


def _probe(debug):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", W4_DEBUG="1" if debug else "0")
    code = PROBE.format(root=ROOT, name="libw4a16_debug.so" if debug else "libw4a16.so",
                        debug=bool(debug))
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-3000:]


def test_debug_library_builds_and_reports_itself():
    lib = build.build(debug=True)
    assert lib.endswith("libw4a16_debug.so") and os.path.exists(lib)
    _probe(debug=True)


def test_normal_library_has_no_checks():
    build.build()
    _probe(debug=False)


def test_checks_compile_away_in_the_normal_build():
    src = open(os.path.join(ROOT, "weight_only_int4_pack_b200", "csrc", "w4_debug.cuh")).read()
    # without W4_DEBUG the macro is a constant true that does not evaluate its condition
    assert "#define W4_CHECK(cond, status) ((void)sizeof(cond), true)" in src
    for f in ("w4_quantize.cu", "w4_decode.cu", "w4_prefill.cu", "w4_gemv.cu", "w4_gemv1.cu"):
        text = open(os.path.join(ROOT, "weight_only_int4_pack_b200", "csrc", f)).read()
        assert len(re.findall(r"W4_CHECK(?:_WARP)?\(", text)) >= 3, f
        assert "__trap" not in text and not re.search(r"(?<!static_)assert\(", text), f
