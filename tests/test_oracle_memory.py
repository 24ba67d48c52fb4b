"""The oracle reads and writes only inside the arrays it is given.

The pin battery of test_oracle_mutations runs against an AddressSanitizer
build of the oracle, in a child process with the sanitizer runtime
preloaded: an access outside any array aborts the child with a report.
The unmodified source must run clean. Each planted off-by-one loop below
changes no value a pin can see (it writes one element past a row, or reads
one past an array), and it must be reported this way.
"""
import os
import subprocess
import sys

import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "pagedkv_oracle.c")
HERE = os.path.dirname(os.path.abspath(__file__))


def _asan_runtime():
    try:
        path = subprocess.run(["gcc", "-print-file-name=libasan.so"], capture_output=True, text=True,
                              check=True).stdout.strip()
    except (OSError, subprocess.CalledProcessError):
        return None
    return path if os.path.isabs(path) and os.path.exists(path) else None


ASAN = _asan_runtime()
pytestmark = pytest.mark.skipif(ASAN is None, reason="gcc's AddressSanitizer runtime is not installed")

MEMORY_MUTANTS = {
    "attention output loop one past the row": (
        "    for (int d = 0; d < head_size; ++d) {\n        double acc = 0.0;\n"
        "        for (int i = 0; i < n; ++i)\n            acc += exp(z[i] - m) * cache_value",
        "d < head_size", "d <= head_size"),
    "empty-context zero fill one past the row": (
        "    if (L <= 0) {\n        for (int d = 0; d < head_size; ++d)\n            o[d] = 0.0;",
        "d < head_size", "d <= head_size"),
    "unused-partition fill one past the row": (
        "                if (p >= nparts) {\n                    for (int d = 0; d < head_size; ++d)",
        "d < head_size", "d <= head_size"),
    "log-sum-exp maximum over one partial too many": (
        "    for (int p = 0; p < n_parts; ++p)\n        if (lse[p] > M)",
        "p < n_parts", "p <= n_parts"),
    "log-sum-exp output loop one past the row": (
        "        wsum += exp(lse[p] - M);\n    for (int d = 0; d < head_size; ++d) {",
        "d < head_size", "d <= head_size"),
    "binary16 array decode one past the end": (
        "void oracle_f16_array_to_double(double *dst, const uint16_t *src, int64_t n)\n{\n"
        "    for (int64_t i = 0; i < n; ++i)",
        "i < n", "i <= n"),
    "E4M3 array encode one past the end": (
        "void oracle_e4m3_array_from_float(uint8_t *dst, const float *src, int64_t n)\n{\n"
        "    for (int64_t i = 0; i < n; ++i)",
        "i < n", "i <= n"),
}

_CHILD = (
    "import sys\n"
    f"sys.path[:0] = [{os.path.dirname(HERE)!r}, {HERE!r}]\n"
    "import oracle, test_oracle_mutations as T\n"
    "with oracle.using_library(sys.argv[1]):\n"
    "    failed = T.pin_battery()\n"
    "sys.exit(1 if failed else 0)\n"
)


def _run_under_asan(source: str, tmp_path) -> tuple[int, str]:
    c = tmp_path / "oracle_asan.c"
    so = tmp_path / "liboracle_asan.so"
    c.write_text(source)
    subprocess.run(["gcc", "-O1", "-g", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
                    "-fsanitize=address", "-fno-omit-frame-pointer", "-shared", "-fPIC", str(c), "-o", str(so),
                    "-lm"], check=True)
    env = dict(os.environ, LD_PRELOAD=ASAN, ASAN_OPTIONS="detect_leaks=0:exitcode=99")
    r = subprocess.run([sys.executable, "-c", _CHILD, str(so)], capture_output=True, text=True, env=env,
                       timeout=600)
    return r.returncode, r.stdout + r.stderr


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


def test_unmodified_oracle_stays_inside_its_arrays(source, tmp_path):
    rc, out = _run_under_asan(source, tmp_path)
    assert "AddressSanitizer" not in out, out[-3000:]
    assert rc == 0, out[-3000:]


@pytest.mark.parametrize("name", sorted(MEMORY_MUTANTS))
def test_planted_out_of_bounds_access_is_reported(source, tmp_path, name):
    anchor, old, new = MEMORY_MUTANTS[name]
    assert source.count(anchor) == 1, f"anchor not unique: {name}"
    rc, out = _run_under_asan(source.replace(anchor, anchor.replace(old, new, 1)), tmp_path)
    assert rc != 0 and "AddressSanitizer" in out, f"not reported: {name}"
