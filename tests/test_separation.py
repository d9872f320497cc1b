"""The CUDA path and the oracle share no code, and the product path has no
CPU fallback (no GPU needed).

* Nothing in the package (Python, CUDA, the C header) imports, loads or
  includes the oracle; the oracle imports nothing from the package and its C
  source includes only the C library.
* The one shared module, the seeded input recipes, imports neither side.
* The package imports with the oracle made unimportable.
* With the CUDA library missing, the binding raises instead of computing
  anything; tensors on the CPU are refused.
"""
import ast
import os
import re
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "nvfp4_w4a4_quantized_act_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for d, _, fs in os.walk(top):
        if "__pycache__" in d:
            continue
        for f in fs:
            if f.endswith(exts):
                yield os.path.join(d, f)


def _imports(path):
    tree = ast.parse(open(path).read(), path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            names.add(("." * node.level) + (node.module or ""))
    return names


def test_package_python_never_imports_the_oracle():
    files = list(_files(PKG, (".py",)))
    assert files
    for path in files:
        for name in _imports(path):
            assert not name.split(".")[0] == "oracle", f"{path} imports {name}"
        text = open(path).read()
        assert "liboracle" not in text and "nvfp4_oracle" not in text, path


def test_cuda_sources_never_include_or_load_the_oracle():
    files = list(_files(os.path.join(PKG, "csrc"), (".cu", ".cuh", ".h", ".cpp"))) + \
        list(_files(os.path.join(ROOT, "include"), (".h",)))
    assert files
    for path in files:
        text = open(path).read()
        for inc in re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', text):
            assert "oracle" not in inc, f"{path} includes {inc}"
        assert "liboracle" not in text and "oracle_" not in text, path


def test_oracle_imports_nothing_from_the_package():
    for path in _files(ORACLE, (".py",)):
        for name in _imports(path):
            assert "nvfp4_w4a4_quantized_act_b200" not in name, f"{path} imports {name}"
    c_src = open(os.path.join(ORACLE, "nvfp4_oracle.c")).read()
    incs = re.findall(r'#\s*include\s*([<"][^>"]+[>"])', c_src)
    assert incs and all(i.startswith("<") for i in incs), incs      # C library headers only


def test_shared_input_recipes_import_neither_side():
    names = _imports(os.path.join(PKG, "workloads.py"))
    for name in names:
        assert name.split(".")[0] != "oracle", name
        assert name.lstrip(".") not in ("ops", "build", "mismatch_report"), name
        assert not name.startswith("nvfp4_w4a4_quantized_act_b200"), name


def _child(code):
    env = dict(os.environ, PYTHONPATH=ROOT, CUDA_VISIBLE_DEVICES="")
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=300)


def test_package_imports_without_the_oracle():
    r = _child("import sys; sys.modules['oracle'] = None\n"
               "import nvfp4_w4a4_quantized_act_b200.ops, nvfp4_w4a4_quantized_act_b200.workloads\n"
               "import nvfp4_w4a4_quantized_act_b200.mismatch_report\n"
               "assert 'oracle' not in [m.split('.')[0] for m in sys.modules if sys.modules[m] is not None]\n"
               "print('ok')")
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr[-2000:]


def test_missing_library_raises():
    r = _child("from nvfp4_w4a4_quantized_act_b200 import ops\n"
               "ops.LIB_PATH = '/nonexistent/libnvfp4.so'\n"
               "ops._lib = None\n"
               "try:\n"
               "    ops.lib()\n"
               "except RuntimeError as e:\n"
               "    print('raised', 'missing' in str(e))\n")
    assert r.returncode == 0 and r.stdout.strip() == "raised True", (r.stdout, r.stderr[-2000:])


@pytest.mark.parametrize("call", ["quantize_act", "fp8_kv_calibrate"])
def test_cpu_tensors_are_refused(call):
    from nvfp4_w4a4_quantized_act_b200 import ops
    with pytest.raises(ValueError, match="CUDA tensors only"):
        getattr(ops, call)(torch.zeros((4, 16), dtype=torch.bfloat16))
