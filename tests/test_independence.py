"""The oracle and the CUDA path stay apart, and the product path has no fallback:
the oracle imports nothing of the package (only the standard library and numpy), no
file of the package imports the oracle, and importing the package without its
compiled library raises instead of falling back to anything."""
import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "qwen3_decoder_block_b200")


def _imports(path):
    tree = ast.parse(open(path, encoding="utf-8").read(), path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name.split(".")[0]
        elif isinstance(node, ast.ImportFrom):
            if node.level == 0 and node.module:
                yield node.module.split(".")[0]


def test_oracle_imports_only_stdlib_and_numpy():
    allowed = {"__future__", "dataclasses", "typing", "math", "numpy", "ctypes", "os", "hashlib", "shutil",
               "subprocess", "sys"}
    for name in os.listdir(os.path.join(ROOT, "oracle")):
        if name.endswith(".py"):
            mods = set(_imports(os.path.join(ROOT, "oracle", name)))
            assert mods <= allowed, (name, mods - allowed)


def test_package_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for name in files:
            path = os.path.join(dirpath, name)
            if name.endswith(".py"):
                assert "oracle" not in set(_imports(path)), path
            elif name.endswith((".cu", ".cuh", ".h")):
                assert "oracle" not in open(path, encoding="utf-8").read(), path


def test_cpp_oracle_includes_nothing_of_the_library():
    src = open(os.path.join(ROOT, "oracle", "qwen3_ref.cpp"), encoding="utf-8").read()
    includes = [l for l in src.splitlines() if l.startswith("#include")]
    assert all("<" in l for l in includes), includes  # standard headers only
    assert "qwen3blk" not in src and "csrc" not in src


def test_package_import_fails_loudly_without_its_library():
    code = (
        "import os, sys\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "real = os.path.exists\n"
        "os.path.exists = lambda p: False if str(p).endswith('libqwen3blk.so') else real(p)\n"
        "try:\n"
        "    import qwen3_decoder_block_b200\n"
        "except ImportError as e:\n"
        "    print('IMPORT_ERROR', e)\n"
        "else:\n"
        "    print('IMPORTED')\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120).stdout
    assert out.startswith("IMPORT_ERROR") and "libqwen3blk.so is missing" in out, out


def test_input_generator_is_a_module_of_its_own():
    """The seeded generator serves both sides and belongs to neither: it imports neither
    the package nor the oracle, and the package does not import it."""
    synth_dir = os.path.join(ROOT, "qwen3_synth")
    for dirpath, _, files in os.walk(synth_dir):
        for name in files:
            if name.endswith(".py"):
                mods = set(_imports(os.path.join(dirpath, name)))
                assert not mods & {"oracle", "qwen3_decoder_block_b200"}, (name, mods)
    for dirpath, _, files in os.walk(PKG):
        for name in files:
            if name.endswith(".py"):
                assert "qwen3_synth" not in set(_imports(os.path.join(dirpath, name))), name


def test_oracle_process_maps_no_product_library():
    """A process that runs the oracle on seeded inputs (what the benchmark's oracle arm
    does) never loads libqwen3blk.so."""
    code = (
        "import sys\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "import numpy as np\n"
        "import oracle.qwen3_ref as R\n"
        "import qwen3_synth as synth\n"
        "x = R.bf16_to_f64(synth.normal_bf16_fast(1, 3, (4, 8)))\n"
        "R.rms_norm(x, np.ones(8), 1e-6)\n"
        "print('LOADED' if 'libqwen3blk' in open('/proc/self/maps').read() else 'CLEAN')\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert out.stdout.strip() == "CLEAN", (out.stdout, out.stderr)
