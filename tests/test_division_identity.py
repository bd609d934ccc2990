"""The quantization kernel divides by E4M3 block scales and by 6 with Markstein's
FMA-corrected quotient instead of a full IEEE division, and the second-level scale
amax / 2688 is a double-precision product rounded to binary32. The FP4 quantizer
evaluates the FMA-corrected quotient two lanes at a time with the reciprocal negated, which
must give exactly the negated quotient (signed zeros included). This checks, on the CPU,
that the identities hold on the domains the kernels use them on (a strided subset here;
the exhaustive run, stride 1, also passes for the first four)."""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.timeout(300)
def test_markstein_quotient_equals_ieee_division(tmp_path):
    exe = str(tmp_path / "div_identity")
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", os.path.join(HERE, "div_identity.c"),
                    "-o", exe, "-lm"], check=True)
    r = subprocess.run([exe, "61"], capture_output=True, text=True)
    print(r.stdout)
    assert r.returncode == 0, r.stdout
