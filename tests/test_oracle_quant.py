"""Pins of the oracle's row-wise 8-bit quantiser (the DLRM_U8ROW table storage):
a hand-worked row, a constant row, the rounding bound |s q + m - v| <= s/2 and
the extreme codes on random rows, and brute force over all 256 codes on small
rows (the pin functions live in pins.py, where the planted-mistake tests also
run them). A floor instead of a round, a wrong offset or a scale off by one
code fails one of them."""
from oracle import oracle as O
from pins import pin_quant_brute_force, pin_quant_constant_row, pin_quant_golden, pin_quant_rounding_bound


def test_worked_example():
    pin_quant_golden(O.load())


def test_constant_row_is_exact():
    pin_quant_constant_row(O.load())


def test_rounding_bound_and_extreme_codes():
    pin_quant_rounding_bound(O.load())


def test_brute_force_nearest_code():
    pin_quant_brute_force(O.load())
