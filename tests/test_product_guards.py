"""The product path: no oracle, no CPU fallback (CPU-only checks)."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(code: str) -> subprocess.CompletedProcess:
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)


def test_product_modules_do_not_import_the_oracle():
    r = _run("import sys\n"
             "import compressed_kv_cache_convkv_b200 as ckv\n"
             "import compressed_kv_cache_convkv_b200.configs, compressed_kv_cache_convkv_b200.sp\n"
             "import compressed_kv_cache_convkv_b200.sharding\n"
             "ckv.library()\n"
             "bad = [m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')]\n"
             "assert not bad, bad\n")
    assert r.returncode == 0, r.stderr


def test_missing_library_fails_loudly():
    r = _run("import compressed_kv_cache_convkv_b200 as ckv\n"
             "ckv.LIB_PATH = '/nonexistent/libconvkv.so'\n"
             "try:\n"
             "    ckv.library()\n"
             "except RuntimeError as e:\n"
             "    print('raised', e)\n"
             "else:\n"
             "    raise SystemExit('no error without the library')\n")
    assert r.returncode == 0 and "raised" in r.stdout, (r.stdout, r.stderr)
