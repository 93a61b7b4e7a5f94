"""The oracle's pins must catch plausible mistakes.

Each case below plants one mistake in a temporary copy of oracle/gdn_oracle.c
(CPU only), builds it with gcc and runs every pin check of test_oracle_pins.py
against it; at least one pin must fail. The committed oracle is never modified.
"""
import os
import subprocess

import pytest

import oracle
from tests.test_oracle_pins import PIN_CHECKS

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

PREFILL_GATE = "    apply_gate(St, exp(c->g[th]), dk, dv);\n"
PREFILL_HH = "    apply_householder(St, kt, c->v + th * dv, c->beta[th], dk, dv);\n"
PREFILL_OUT = "    emit_output(St, qt, c->scale, c->o + th * dv, dk, dv);\n"

MUTANTS = {
    # the gate scales the token's own write (gate after the update)
    "gate_after_update": [(PREFILL_GATE + PREFILL_HH, PREFILL_HH + PREFILL_GATE)],
    # the output is read before the token's update
    "output_before_update": [(PREFILL_GATE + PREFILL_HH + PREFILL_OUT,
                              PREFILL_OUT + PREFILL_GATE + PREFILL_HH)],
    # beta dropped from the write term
    "write_without_beta": [("+ beta * k[i] * v[j]", "+ k[i] * v[j]")],
    # wrong sign of the projection term
    "projection_sign": [("col[i] - beta * k[i] * p", "col[i] + beta * k[i] * p")],
    # output contracts the transposed state
    "output_transposed": [(
        "    const double* col = St + (size_t)j * dk;\n    double acc = 0.0;\n"
        "    for (int i = 0; i < dk; ++i) acc += col[i] * q[i];",
        "    double acc = 0.0;\n"
        "    for (int i = 0; i < dk; ++i) acc += St[(size_t)i * dv + j] * q[i];")],
    # scale not applied
    "no_scale": [("o[j] = scale * acc;", "o[j] = acc;")],
    # gate linearised (alpha = 1 + g instead of exp(g))
    "gate_linearised": [("apply_gate(St, exp(c->g[th]), dk, dv);", "apply_gate(St, 1.0 + c->g[th], dk, dv);"),
                        ("apply_gate(St, exp(c->g[bth]), dk, dv);", "apply_gate(St, 1.0 + c->g[bth], dk, dv);")],
    # gated delta product: the gate applied before every Householder update
    "gdp_gate_per_householder": [(
        "    apply_gate(St, exp(c->g[bth]), dk, dv);\n    for (int m = 0; m < nh; ++m) {\n",
        "    for (int m = 0; m < nh; ++m) {\n      apply_gate(St, exp(c->g[bth]), dk, dv);\n")],
    # gated delta product: Householder updates applied in reverse order
    "gdp_reverse_order": [("      const size_t km = bth * nh + m;", "      const size_t km = bth * nh + (nh - 1 - m);")],
    # the projection uses the previous token's key
    "stale_key": [("const double* kt = maybe_unit(c->k + tq * dk,",
                   "const double* kt = maybe_unit(c->k + (t > c->cu[n] ? tq - Hqk : tq) * dk,")],
    # grouped heads: value head h reads q/k head h % H_qk instead of h / (H / H_qk)
    "grouped_heads_modulo": [("  const int hq = h / (H / Hqk); /* the value head's query/key head */\n"
                              "  const size_t ssz",
                              "  const int hq = h % Hqk;\n  const size_t ssz"),
                             ("  const int hq = h / (H / Hqk); /* the value head's query/key head */\n"
                              "  const int slot",
                              "  const int hq = h % Hqk;\n  const int slot")],
    # the q/k normalisation applied to the query only
    "l2norm_query_only": [("const double* kt = maybe_unit(c->k + tq * dk, dk, c->l2norm, buf);",
                           "const double* kt = c->k + tq * dk;")],
    # the per-token state recorded before the token's update instead of after it
    "token_state_before_update": [(
        "    if (c->token_states) /* the state after token t (speculative-verify rollback point) */\n"
        "      memcpy(c->token_states + bth * (size_t)dk * dv, St, (size_t)dk * dv * sizeof(double));\n",
        ""), (
        "    apply_gate(St, exp(c->g[bth]), dk, dv);\n    for (int m = 0; m < nh; ++m) {\n",
        "    if (c->token_states)\n"
        "      memcpy(c->token_states + bth * (size_t)dk * dv, St, (size_t)dk * dv * sizeof(double));\n"
        "    apply_gate(St, exp(c->g[bth]), dk, dv);\n    for (int m = 0; m < nh; ++m) {\n")],
    # the normalisation divides by the squared norm
    # backward: the key derivative without its state term
    "backward_dk_without_state_term": [("dkv[i] = beta * (a - b);", "dkv[i] = beta * a;")],
    # backward: wrong sign of the Householder part of the gate derivative
    "backward_dg_sign": [("c->dg[th] = ds - beta * uw;", "c->dg[th] = ds + beta * uw;")],
    # backward: the state derivative carried to the previous token without the gate
    "backward_carry_without_gate": [("Dt[(size_t)j * dk + i] = alpha * (Dt[(size_t)j * dk + i] - beta * k[i] * w[j]);",
                                     "Dt[(size_t)j * dk + i] = Dt[(size_t)j * dk + i] - beta * k[i] * w[j];")],
    # backward: the query derivative read from the previous state
    "backward_dq_previous_state": [("acc += St[(size_t)j * dk + i] * dO[j];", "acc += Sp[(size_t)j * dk + i] * dO[j];")],
    # backward: the normalisation's derivative without its projection term
    "backward_l2norm_without_projection": [("for (int i = 0; i < n; ++i) d[i] = (d[i] - x[i] * inv * dot) * inv;",
                                            "for (int i = 0; i < n; ++i) d[i] = d[i] * inv;")],
    "l2norm_squared": [("const double inv = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;",
                        "const double inv = ss > 0.0 ? 1.0 / ss : 0.0;")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    src = open(SRC).read()
    for old, new in MUTANTS[name]:
        assert old in src, f"mutation anchor not found for {name}: {old!r}"
        src = src.replace(old, new)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "libmutant.so"
    c_path.write_text(src)
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c99", "-D_POSIX_C_SOURCE=200809L",
                           "-o", str(so_path), str(c_path), "-lm", "-lpthread"])
    lib = oracle.load_library(str(so_path))
    failed = []
    for check in PIN_CHECKS:
        try:
            check(lib)
        except (AssertionError, ValueError):
            failed.append(check.__name__)
    assert failed, f"no pin caught mutant {name}"
