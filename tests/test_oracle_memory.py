"""Pins for per-rank model-state accounting and logical communication volume:
the pages' closed forms and the worked numbers they print."""
import json
import os

import pytest

import oracle
from synth import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "memory_examples.json")
KEY = {"dp": oracle.STAGE_DP, "zero1": oracle.STAGE_Z1, "zero2": oracle.STAGE_Z2,
       "zero3": oracle.STAGE_Z3}


def test_bytes_per_param_is_16():
    g = json.load(open(GOLDEN))["bytes_per_param"]
    assert g["param16"] + g["grad16"] + g["master32"] + g["m32"] + g["v32"] == g["total"] == 16
    assert oracle.mem_model(1.0, 1)[oracle.STAGE_DP] == g["total"]


@pytest.mark.parametrize("example", json.load(open(GOLDEN))["examples"])
def test_worked_examples_to_printed_digits(example):
    model = oracle.mem_model(example["psi"], example["n_ranks"])
    for name, gb in example["per_card_gb"].items():
        digits = example["printed_digits"][name]
        assert round(model[KEY[name]] / 1e9, digits) == pytest.approx(gb, abs=1e-9), name


@pytest.mark.parametrize("n_ranks", [1, 2, 4, 8, 16, 64])
def test_closed_forms(n_ranks):
    """Per-rank state bytes from the plan equal 16P, 4P + 12P/N, 2P + 14P/N,
    16P/N exactly when the parameter count needs no padding."""
    numel, layer = W.transformer_layers(4, 128, 512)  # 793,088 = 1549 * 512 params
    p = oracle.plan(numel, layer, n_ranks, 1 << 16)
    P = p.psi
    assert p.psi_pad == P
    forms = {oracle.STAGE_DP: 16 * P, oracle.STAGE_Z1: 4 * P + 12 * P // n_ranks,
             oracle.STAGE_Z2: 2 * P + 14 * P // n_ranks, oracle.STAGE_Z3: 16 * P // n_ranks}
    for stage, want in forms.items():
        assert sum(oracle.state_bytes(p, stage)) == want
        assert oracle.mem_model(P, n_ranks)[stage] == pytest.approx(want, rel=1e-15)


@pytest.mark.parametrize("n_ranks", [2, 4, 8, 64])
def test_zero3_moves_one_and_a_half_times_allreduce(n_ranks):
    g = json.load(open(GOLDEN))["zero3_comm_vs_allreduce"]
    p = oracle.plan([n_ranks * 8 * 1000], [0], n_ranks, 1 << 20)
    vol = {s: sum(oracle.comm_elems(p, s).values()) for s in range(4)}
    assert vol[oracle.STAGE_Z3] / vol[oracle.STAGE_DP] == g["ratio"]
    assert vol[oracle.STAGE_Z2] == vol[oracle.STAGE_DP]          # RS + AG = AR
    assert vol[oracle.STAGE_Z1] / vol[oracle.STAGE_DP] == 1.5    # AR then AG


def test_workload_parameter_counts():
    assert W.flat_1m_n4().psi == 1_048_576
    assert W.gpt_85m_n8().psi == 85_054_464
    assert W.gpt_1p2b_n8().psi == 1_208_598_528
    assert W.gpt_6p4b_n64().psi == 6_444_154_880
