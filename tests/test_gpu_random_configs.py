"""A seeded sweep of random small layer configurations (tests/random_configs.py)
through moe_forward / moe_forward_ex against the fp64 oracle, cycling the
launch forms: single launch in static and dynamic tile order, two launches,
CTA pairs in both, four-box B copies, and the gate_up GEMM gathering its
own rows (row f1) in one and in two launches. Same bars as every parity test:
routing bit-exact, router weights 1e-5 relative, output 2e-2 * max|ref|."""
import pytest

from gpu_helpers import run_and_check, run_and_check_ex
from random_configs import NUM_CASES, random_workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("i", range(NUM_CASES))
def test_random_config(i, monkeypatch):
    wl, form = random_workload(i)
    for key, value in form.items():
        monkeypatch.setenv(key, value)
    if wl.extended:
        run_and_check_ex(wl, seed=i)
    else:
        run_and_check(wl, seed=i)
