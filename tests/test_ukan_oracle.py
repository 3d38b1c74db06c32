"""The UKAN oracle (oracle/ukan.py) against its pins (CPU only), and mutants of it against the same pins."""
import importlib.util
import sys

import pytest

import pins_ukan
from oracle import ukan


@pytest.mark.parametrize("pin", pins_ukan.ALL_PINS, ids=lambda p: p.__name__)
def test_ukan_pin(pin):
    assert pin(ukan) is None


MUTANTS = {
    "sin_cos_swapped": ("pe[:, 0::2] = np.sin(q * w)\n    pe[:, 1::2] = np.cos(q * w)",
                        "pe[:, 0::2] = np.cos(q * w)\n    pe[:, 1::2] = np.sin(q * w)"),
    "group_offset": ("m0 = q0 * g\n    for m_loc in range(nq * g):\n        B, _ = basis(x, m0 + m_loc, h)",
                     "m0 = q0 * g\n    for m_loc in range(nq * g):\n        B, _ = basis(x, m0 + m_loc + 1, h)"),
    "dsilu_wrong": ("return s * (1.0 + z * (1.0 - s))", "return s * (1.0 - z * (1.0 - s))"),
    "edge_layout": ("c.reshape(nq, n_out, n_in, g).transpose(1, 2, 0, 3)", "c.reshape(nq, n_in, n_out, g).transpose(2, 1, 0, 3)"),
    "derivative_shift": ("(cardinal(v, 2) - cardinal(v - 1.0, 2)) / h", "(cardinal(v, 2) - cardinal(v + 1.0, 2)) / h"),
    "db1_missing_dsilu": ("dpre = (dc @ W2) * dsilu(pre)", "dpre = (dc @ W2) * silu(pre)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_ukan_mutant_is_caught(tmp_path, name):
    src = open(ukan.__file__).read()
    before, after = MUTANTS[name]
    assert src.count(before) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / f"ukan_{name}.py"
    path.write_text(src.replace(before, after))
    spec = importlib.util.spec_from_file_location(f"ukan_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    assert pins_ukan.run_all(mod), f"mutant {name} passed every pin"
