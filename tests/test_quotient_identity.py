"""The identity the GPU quantizer relies on instead of dividing per element
(Markstein's correction of the quotient from the row's reciprocal), checked
on the host in plain C (tests/quotient_identity.c) against IEEE division:
every bf16 value below every 16th positive bf16 row maximum, for the int8
(127) and E4M3 (448) scales, and fp32 values planted at and around every
half-integer quotient of pseudo-random scales.  The full sweep
(`quotient_identity 1 100000`: every bf16 row maximum, 3.6 * 10^9 checks,
about a minute and a half) passes as well; this test keeps a sixteenth of
the bf16 part."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("quotient") / "quotient_identity")
    subprocess.run([cc, "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-o", exe,
                    os.path.join(HERE, "quotient_identity.c"), "-lm"], check=True)
    return exe


def test_markstein_quotient_equals_ieee_division(checker):
    out = subprocess.run([checker, "16", "2000"], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout[-2000:]
    assert "mismatches 0" in out.stdout, out.stdout


def test_checker_detects_an_uncorrected_quotient(tmp_path):
    """The checker itself fails on the plain product fl32(x * r) (no
    correction): it is able to see a wrong quotient."""
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = open(os.path.join(HERE, "quotient_identity.c")).read()
    site = "  return fmaf(e, r, q0);\n"
    assert src.count(site) == 1
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(site, "  (void)e;\n  return q0;\n"))
    exe = str(tmp_path / "mutant")
    subprocess.run([cc, "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-o", exe, str(mutant), "-lm"],
                   check=True)
    out = subprocess.run([exe, "64", "50"], capture_output=True, text=True, timeout=600)
    assert out.returncode == 1 and "mismatches 0" not in out.stdout, out.stdout
