"""Oracle pins: masked attention and block mass (CPU only)."""
from oracle import attention, lvsa
from tests import pins


def test_vs_torch_sdpa_f64():
    pins.check_attention_vs_sdpa(attention, lvsa)


def test_closed_forms():
    pins.check_attention_closed_forms(attention, lvsa)


def test_triple_loop():
    pins.check_attention_triple_loop(attention, lvsa)


def test_block_mass():
    pins.check_block_mass(attention)


def test_block_mass_restricted():
    pins.check_block_mass_restricted(attention, lvsa)
