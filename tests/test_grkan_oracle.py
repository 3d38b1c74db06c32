"""The GR-KAN oracle (oracle/grkan.py) against its pins (CPU only), and mutants of it against the same pins."""
import importlib.util
import sys

import pytest

import pins_grkan
from oracle import grkan


@pytest.mark.parametrize("pin", pins_grkan.ALL_PINS, ids=lambda p: p.__name__)
def test_grkan_pin(pin):
    assert pin(grkan) is None


# Each plausible mistake, planted in a private copy of the oracle source on the CPU, must make at
# least one pin fail.
MUTANTS = {
    "missing_abs": ("Q = 1.0 + np.abs(S)\n        phi", "Q = 1.0 + S\n        phi"),
    "forward_missing_abs": ("return P / (1.0 + np.abs(S))", "return P / (1.0 + S)"),
    "dx_sign": ("gs * (dP - phi * sg * dS) / Q", "gs * (dP + phi * sg * dS) / Q"),
    "dx_missing_q": ("gs * (dP - phi * sg * dS) / Q", "gs * (dP - phi * sg * dS)"),
    "db_sign": ("gb = -gs * phi * sg / Q", "gb = gs * phi * sg / Q"),
    "da_square": ("ga = gs / Q  ", "ga = gs / Q**2"),
    "interleaved_groups": ("gi = np.arange(C) // cg", "gi = np.arange(C) % groups"),
    "db_power_off_by_one": ("xp = xg.copy()", "xp = np.ones_like(xg)"),
    "derivative_coefficients": ("dA = A[:, 1:] * np.arange(1, m + 1)", "dA = A[:, 1:]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_grkan_mutant_is_caught(tmp_path, name):
    src = open(grkan.__file__).read()
    before, after = MUTANTS[name]
    assert src.count(before) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / f"grkan_{name}.py"
    path.write_text(src.replace(before, after))
    spec = importlib.util.spec_from_file_location(f"grkan_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    assert pins_grkan.run_all(mod), f"mutant {name} passed every pin"
