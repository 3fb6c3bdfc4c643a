"""A few planted mistakes from ``tests/oracle_mutants.py`` run in the CPU
suite: each must make the oracle's tests fail.  The full list (58 mutants,
a few minutes) runs with ``python tests/oracle_mutants.py WORKDIR``."""
import pytest

from tests import oracle_mutants as om

SMOKE = ("encode_block ties to larger", "pack low nibble first", "DQ fp32 ratio", "dX sign",
         "bf16 subnormal threshold", "int4 ties to even", "decode fused")


def test_smoke_mutants_are_caught(tmp_path):
    om._copy(str(tmp_path))
    assert om._run(str(tmp_path)), "the unmodified oracle must pass its tests"
    by_name = {m[3]: m for m in om.MUTANTS}
    for name in SMOKE:
        fn, old, new, _ = by_name[name]
        path = tmp_path / "oracle" / fn
        src = path.read_text()
        assert src.count(old) == 1, name
        path.write_text(src.replace(old, new))
        try:
            assert not om._run(str(tmp_path)), f"planted mistake not caught: {name}"
        finally:
            path.write_text(src)


def test_expected_survivors_are_listed():
    names = {m[3] for m in om.MUTANTS}
    assert om.EXPECTED_SURVIVORS <= names
    assert len(names) == len(om.MUTANTS)
