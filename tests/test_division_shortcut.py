"""The quantiser's block-scale quotient shortcut (hoisted reciprocal + one exact FMA correction)
yields the same E4M3 block-scale code as the correctly rounded division wherever the kernel uses
it; where the kernel falls back to the division (tiny block maxima) the shortcut alone would not."""
import os
import shutil
import subprocess

import pytest

SRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "c", "block_scale_quotient.c")


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    out = str(tmp_path_factory.mktemp("bsq") / "bsq")
    subprocess.run([cc, "-O2", "-ffp-contract=off", "-o", out, SRC, "-lm"], check=True)
    return out


def _run(exe, n, guard, target=6):
    text = subprocess.run([exe, str(n), str(guard), str(target)], check=True, capture_output=True,
                          text=True).stdout
    _, tested, _, mism = text.split()
    return int(tested), int(mism)


def test_shortcut_matches_division_codes_where_the_kernel_uses_it(exe):
    tested, mism = _run(exe, 600, 1)
    assert tested > 5_000_000
    assert mism == 0


def test_the_tiny_block_guard_is_needed(exe):
    _, mism = _run(exe, 600, 0)
    assert mism > 0


@pytest.mark.parametrize("target", [6, 4])
def test_shortcut_matches_division_codes_for_every_bf16_chunk_maximum(exe, target):
    # every positive finite bf16 chunk maximum A and every bf16 block maximum a <= A, for the
    # scale target 6 and the adaptive candidate's target 4
    tested, mism = _run(exe, 0, 1, target)
    assert tested > 400_000_000
    assert mism == 0
