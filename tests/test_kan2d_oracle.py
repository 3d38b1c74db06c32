"""The 2-D (tensor-product surface) oracle against its pins (CPU only), and mutants of it."""
import importlib.util
import sys

import pytest

import pins_2d
from oracle import kan2d


def test_2d_pins(oracle):
    assert pins_2d.pin_marsden(kan2d) is None
    assert pins_2d.pin_marsden(kan2d, k=2) is None
    assert pins_2d.pin_partition(kan2d) is None
    assert pins_2d.pin_reduces_to_1d(kan2d, oracle) is None
    assert pins_2d.pin_finite_difference(kan2d) is None
    assert pins_2d.pin_linear(kan2d) is None


MUTANTS = {
    "swapped_coordinates": ("Bu, Bv = B[:, 0::2], B[:, 1::2]", "Bu, Bv = B[:, 1::2], B[:, 0::2]"),
    "transposed_surface": ('"bpm,bpn,jpmn->bj"', '"bpm,bpn,jpnm->bj"'),
    "dx_v_derivative_on_u": ('dx[:, 1::2] = np.einsum("bpmn,bpm,bpn->bp", Gm, Bu, dBv',
                             'dx[:, 1::2] = np.einsum("bpmn,bpm,bpn->bp", Gm, dBu, Bv'),
    "dcoef_transposed": ('"bj,bpm,bpn->jpmn"', '"bj,bpm,bpn->jpnm"'),
    "dx_u_without_v": ('dx[:, 0::2] = np.einsum("bpmn,bpm,bpn->bp", Gm, dBu, Bv',
                       'dx[:, 0::2] = np.einsum("bpmn,bpm,bpn->bp", Gm, dBu, dBv'),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_2d_mutant_is_caught(tmp_path, oracle, name):
    src = open(kan2d.__file__).read()
    before, after = MUTANTS[name]
    assert src.count(before) == 1, f"mutation anchor for {name} not found exactly once"
    src = src.replace(before, after).replace("from . import get as _get_1d", "from oracle import get as _get_1d")
    path = tmp_path / f"kan2d_{name}.py"
    path.write_text(src)
    spec = importlib.util.spec_from_file_location(f"kan2d_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    assert pins_2d.run_all(mod, oracle), f"mutant {name} passed every pin"
