"""Planted mistakes in a copy of the oracle must fail its pins (CPU).

Each case copies the oracle (its C++ source and ctypes wrapper) into a
temporary directory, plants one plausible mistake in the source, builds the
copy, and runs the oracle's pin suites against it in a child process. The case
passes only if some pin fails. A control case runs the same harness on the
unmodified copy, which must pass. What this checks is the pins, not the
oracle: a pin set that let one of these through would not pin the oracle.
The mistakes are the ones such code is prone to: a dropped scale, an
off-by-one or misaligned mask, a missing max subtraction or normalisation, the
wrong log base, transposed or shifted indices, the wrong exponent bias, a
wrong head mapping, and a dropped or wrong term in the gradients.
"""

import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["tests/test_oracle_pins.py", "tests/test_oracle_varlen_pins.py", "tests/test_oracle_backward_pins.py",
             "tests/test_oracle_backward_varlen_pins.py"]

# (name, text in attention_oracle.cpp, replacement, which occurrence: 0 = first only)
MUTANTS = [
    ("dropped_scale", "s[j] = p.scale * dot;", "s[j] = dot;"),
    ("causal_off_by_one", "return p.causal ? (i + 1) : p.N;", "return p.causal ? i : p.N;"),
    ("no_max_subtraction", "e[j] = std::exp(s[j] - m);", "e[j] = std::exp(s[j]);"),
    ("lse_log2", "return m + std::log(l);", "return m + std::log2(l);"),
    ("reversed_v_rows", "const double* vj = &V[j * p.D];", "const double* vj = &V[(nvis - 1 - j) * p.D];"),
    ("shifted_k_index", "dot += qi[d] * kj[d];", "dot += qi[d] * kj[(d + 1) % p.D];"),
    ("fp16_exponent_bias", "mag = std::ldexp(static_cast<double>(1024 + f), e - 25);",
     "mag = std::ldexp(static_cast<double>(1024 + f), e - 24);"),
    ("no_normalisation", "for (int64_t d = 0; d < p.D; ++d) o_out[d] = acc[d] / l;",
     "for (int64_t d = 0; d < p.D; ++d) o_out[d] = acc[d];"),
    ("varlen_top_left_mask", "if (causal) nvis = std::min(nk, std::max<int64_t>(0, i + nk - nq + 1));",
     "if (causal) nvis = std::min(nk, std::max<int64_t>(0, i + 1));"),
    ("varlen_interleaved_heads", "const int64_t hk = h / group;", "const int64_t hk = h % Hkv;"),
    ("ds_without_delta", "dS[i * N + j] = pij * (dpij - Di);", "dS[i * N + j] = pij * dpij;"),
    ("dk_without_scale", "dk[at(p, b, j, h, d)] = scale * ak;", "dk[at(p, b, j, h, d)] = ak;"),
    ("dv_from_ds", "av += P[i * N + j] * dO[i * D + d];", "av += dS[i * N + j] * dO[i * D + d];"),
    ("delta_without_o", "for (int64_t d = 0; d < D; ++d) Di += dO[i * D + d] * orow[d];",
     "for (int64_t d = 0; d < D; ++d) Di += dO[i * D + d];"),
    ("backward_mask_off_by_one", "if (j < nvis) {", "if (j <= nvis) {"),
]


def _make_copy(dst, mutation=None):
    """A minimal tree (oracle, input recipe, pin suites) with at most one planted mistake."""
    os.makedirs(os.path.join(dst, "oracle"))
    for f in ("__init__.py", "attention_oracle.cpp"):
        shutil.copy(os.path.join(ROOT, "oracle", f), os.path.join(dst, "oracle", f))
    pkg = os.path.join(dst, "exact_attention_151_b200")
    os.makedirs(pkg)
    for f in os.listdir(os.path.join(ROOT, "exact_attention_151_b200")):
        if f.endswith(".py"):
            shutil.copy(os.path.join(ROOT, "exact_attention_151_b200", f), os.path.join(pkg, f))
    tests = os.path.join(dst, "tests")
    os.makedirs(tests)
    for f in ["__init__.py", "conftest.py", "parity.py"] + [os.path.basename(p) for p in PIN_FILES]:
        if os.path.exists(os.path.join(ROOT, "tests", f)):
            shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(tests, f))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(tests, "golden"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), os.path.join(dst, "pytest.ini"))
    if mutation is not None:
        path = os.path.join(dst, "oracle", "attention_oracle.cpp")
        src = open(path).read()
        old, new = mutation
        assert old in src, f"mutation target no longer in the oracle source: {old}"
        open(path, "w").write(src.replace(old, new, 1))


def _run_pins(dst):
    """Build the copy, then run the pin suites in it; returns (build ok, pytest return code, tail)."""
    b = subprocess.run(["g++", "-std=c++17", "-O2", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC",
                        "-pthread", os.path.join(dst, "oracle", "attention_oracle.cpp"), "-o",
                        os.path.join(dst, "oracle", "liboracle.so")], capture_output=True, text=True)
    if b.returncode != 0:
        return False, None, b.stderr[-500:]
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", *PIN_FILES, "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu"], cwd=dst, capture_output=True, text=True, timeout=600, env=env)
    return True, r.returncode, (r.stdout + r.stderr)[-800:]


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    jobs = {"control": None, **{name: (old, new) for name, old, new in MUTANTS}}
    dirs = {}
    for name, mut in jobs.items():
        d = str(tmp_path_factory.mktemp(name))
        os.rmdir(d)
        _make_copy(d, mut)
        dirs[name] = d
    workers = max(1, min(8, os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        futs = {name: ex.submit(_run_pins, d) for name, d in dirs.items()}
        return {name: f.result() for name, f in futs.items()}


def test_unmodified_copy_passes_its_pins(results):
    built, rc, tail = results["control"]
    assert built and rc == 0, tail


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(results, name):
    built, rc, tail = results[name]
    assert built, tail           # the mutant compiles: it is a wrong oracle, not a broken one
    assert rc == 1, tail         # pytest's code for "some test failed" (not a collection or usage error)
    assert " failed" in tail, tail
