"""The oracle's pins are strong enough to catch plausible mistakes.

Each case plants one mistake in a temporary copy of oracle.c (on the CPU),
builds it, runs the pin suite against that build and expects at least one
pin to fail.  The real oracle is untouched.
"""
import os
import subprocess
import tempfile

import pytest

import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "oracle.c")

MUTANTS = {
    "relu_dropped": ("double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;"),
    "w_wrong_head": ("I += (double)w[(int64_t)t * HI + h] * relu;", "I += (double)w[(int64_t)t * HI] * relu;"),
    "k_dims_shifted": ("dot += q[h * DI + d] * orc_e4m3_to_f64(k[d]);",
                       "dot += q[h * DI + d] * orc_e4m3_to_f64(k[(d + 1) % DI]);"),
    "q_head_transposed": ("dot += q[h * DI + d] * orc_e4m3_to_f64(k[d]);",
                          "dot += q[d * HI % (HI * DI) + h] * orc_e4m3_to_f64(k[d]);"),
    "causal_off_by_one": ("for (int64_t s = 0; s <= p; ++s) {", "for (int64_t s = 0; s < p; ++s) {"),
    "page_table_ignored": ("return (int64_t)page * page_size + pos % page_size;",
                           "return lp * page_size + pos % page_size;"),
    "tie_to_higher_pos": ("return (x->pos < y->pos) ? -1 : (x->pos > y->pos);",
                          "return (x->pos > y->pos) ? -1 : (x->pos < y->pos);"),
    "ascending_scores": ("if (x->v > y->v) return -1;\n    if (x->v < y->v) return 1;",
                         "if (x->v < y->v) return -1;\n    if (x->v > y->v) return 1;"),
    "gate_dropped": ("for (int d = 0; d < Dv; ++d) o[d] *= sig;", "for (int d = 0; d < Dv; ++d) o[d] *= 1.0;"),
    "gate_not_sigmoid": ("double sig = 1.0 / (1.0 + exp(-g));", "double sig = g;"),
    "scale_dropped": ("lg[j] = sm_scale * dot;", "lg[j] = dot;"),
    "value_rows_shifted": ("for (int d = 0; d < Dv; ++d) o[d] += p * orc_bf16_to_f64(c[d]);",
                           "for (int d = 0; d < Dv; ++d) o[d] += p * orc_bf16_to_f64(c[Dqk - Dv + d]);"),
    "e4m3_bias": ("else        v = ldexp(1.0 + (double)m / 8.0, e - 7);",
                  "else        v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "swa_window_short": ("int64_t p0 = L - W > 0 ? L - W : 0;", "int64_t p0 = L - W + 1 > 0 ? L - W + 1 : 0;"),
    "swa_wrong_slot": ("int64_t slot = (p0 + i) % W;\n                const uint16_t *k",
                       "int64_t slot = i % W;\n                const uint16_t *k"),
    "e4m3_ties_away": ("double q = nearbyint(ldexp(a, 3 - e)); /* in [8, 16] */",
                       "double q = round(ldexp(a, 3 - e)); /* in [8, 16] */"),
    "e4m3_no_saturation": ("if (a >= 448.0) return s | 0x7E;", "if (a >= 480.0) return s | 0x7F;"),
    "append_scale_after_rounding": ("float x = (float)orc_bf16_to_f64(k_new[(int64_t)j * DI + d]) * k_scale;",
                                    "float x = (float)orc_e4m3_to_f64(orc_e4m3_from_f64(orc_bf16_to_f64("
                                    "k_new[(int64_t)j * DI + d]))) * k_scale;"),
    "mx_emax_off_by_one": ("shared = (E - 1) - 8;", "shared = (E - 1) - 7;"),
    "mx_low_clamp_wrong": ("if (shared < -127) shared = -127;", "if (shared < -126) shared = -126;"),
    "mx_q_scale_ignores_head": ("int64_t sc = ((int64_t)t * HI + h) * nb + d / ORC_MX_BLOCK;",
                                "int64_t sc = (int64_t)t * nb + d / ORC_MX_BLOCK;"),
    "mx_k_scale_wrong_block": ("orc_e8m0_to_f64(ks[d / ORC_MX_BLOCK])", "orc_e8m0_to_f64(ks[d % nb])"),
    "mx_k_scale_dropped": ("(orc_e4m3_to_f64(k[d]) * orc_e8m0_to_f64(ks[d / ORC_MX_BLOCK]))", "orc_e4m3_to_f64(k[d])"),
    "mx_append_scale_row": ("k_scales + r * nb + blk))", "k_scales + (int64_t)j * nb + blk))"),
}

PIN_TESTS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _pin_calls(fn, orc):
    """The keyword sets pytest would call a pin with: orc, and each value of
    its (single-argument) parametrize marks."""
    import inspect
    base = {"orc": orc} if "orc" in inspect.signature(fn).parameters else {}
    calls = [base]
    for mark in getattr(fn, "pytestmark", []):
        if mark.name == "parametrize":
            name, values = mark.args[0], mark.args[1]
            calls = [dict(c, **{name: v}) for c in calls for v in values]
    return calls


def _pin_failures(orc):
    failed = []
    for fn in PIN_TESTS:
        for kw in _pin_calls(fn, orc):
            try:
                fn(**kw)
            except Exception:
                failed.append(f"{fn.__name__}{sorted((k, v) for k, v in kw.items() if k != 'orc')}")
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(orc, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "m.c")
        so = os.path.join(d, "m.so")
        open(c, "w").write(mutated)
        subprocess.check_call(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", so, c, "-lm"])
        with orc.use_library(so):
            failed = _pin_failures(orc)
    assert failed, f"no pin caught the planted mistake '{name}'"


def test_unmutated_oracle_passes_every_pin(orc):
    assert _pin_failures(orc) == []


# ---- the context-parallel decode oracle (Python): planted in a copy of oracle.py

PY_SRC = os.path.join(os.path.dirname(SRC), "oracle.py")

PY_MUTANTS = {
    "cp_ties_to_higher_position": ("order = np.lexsort((p, -s.astype(np.float64)))[:K]",
                                   "order = np.lexsort((-p, -s.astype(np.float64)))[:K]"),
    "cp_merge_unweighted": ("out = (wgt[..., None] * np.stack(outs)).sum(axis=0)",
                            "out = (np.stack(outs) * (wgt[..., None] > 0)).sum(axis=0)"),
    "cp_local_positions_not_offset": ("cand_p[b].append(sel.astype(np.int64) + lo[b])",
                                      "cand_p[b].append(sel.astype(np.int64))"),
    "cp_rank_misses_its_last_position": ("(n[live] - 1).astype(np.int32), ld=ld)",
                                         "np.maximum(n[live] - 2, 0).astype(np.int32), ld=ld)"),
}


def _cp_pin_failures(mod):
    runs = [(pins.test_context_parallel_decode_is_the_single_device_layer, {}),
            (pins.test_context_parallel_decode_breaks_threshold_ties_across_ranks_by_position, {"w_sign": 1.0}),
            (pins.test_context_parallel_decode_breaks_threshold_ties_across_ranks_by_position, {"w_sign": -1.0})]
    failed = []
    for fn, kw in runs:
        try:
            fn(orc=mod, **kw)
        except Exception:
            failed.append(fn.__name__)
    return failed


def _py_module(src):
    import types
    mod = types.ModuleType("oracle_variant")
    mod.__file__ = PY_SRC
    exec(compile(src, PY_SRC, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_planted_mistake_in_the_context_parallel_oracle_is_caught(name):
    old, new = PY_MUTANTS[name]
    src = open(PY_SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found"
    assert _cp_pin_failures(_py_module(src.replace(old, new, 1))), f"no pin caught '{name}'"


def test_unmutated_context_parallel_oracle_passes_its_pins():
    assert _cp_pin_failures(_py_module(open(PY_SRC).read())) == []
