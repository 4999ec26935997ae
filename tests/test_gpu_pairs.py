"""Both grouped-GEMM schedules against the oracle: single CTAs with 128-row
tiles and CTA pairs (cta_group::2) with 256-row tiles split 128/128, whose
leader issues the MMAs for both.  The library picks one by rows per expert;
MOE_B200_PAIR forces it."""

import numpy as np
import pytest

from gpu_helpers import TOL, f64, i64, oracle_for, rel, run_layer
from test_gpu_layer import CASES

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["0", "1"])
@pytest.mark.parametrize("name", ["bf16_e8_small", "bf16_skew_small", "bf16_dense", "bf16_e128_small"])
def test_gemm_schedule_matches_oracle(name, mode, monkeypatch):
    monkeypatch.setenv("MOE_B200_PAIR", mode)
    cfg = CASES[name]
    cpu, L = run_layer(cfg)
    o = oracle_for(cpu, L)
    assert np.array_equal(i64(L.offsets), o["offsets"])
    R, f = cfg.R, cfg.d_ff
    act = f64(L.act[:R])
    checks = {"a": (act[:, :f], o["a"]), "u": (act[:, f:2 * f], o["u"]), "h": (act[:, 2 * f:], o["h"]),
              "y_perm": (f64(L.y_perm[:R]), o["y_perm"]), "dx_perm": (f64(L.dx_perm[:R]), o["dx_perm"]),
              "out": (f64(L.out), o["out"]), "dx": (f64(L.dx), o["dx"]),
              "dw1": (f64(L.dw1), o["dw1"]), "dw2": (f64(L.dw2), o["dw2"])}
    errs = {k: rel(a, b) for k, (a, b) in checks.items()}
    assert all(v <= TOL["bf16"] for v in errs.values()), (name, mode, errs)


@pytest.mark.parametrize("capacity", [40])
def test_padded_layout_with_pairs(capacity, monkeypatch):
    monkeypatch.setenv("MOE_B200_PAIR", "1")
    cfg = CASES["bf16_skew_small"]
    cpu, L = run_layer(cfg, capacity=capacity)
    o = oracle_for(cpu, L, capacity=capacity)
    for key, dev in (("out", L.out), ("dx", L.dx), ("dw1", L.dw1), ("dw2", L.dw2)):
        assert rel(f64(dev), o[key]) <= TOL["bf16"], key
