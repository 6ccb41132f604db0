"""The model-level oracle against the hand-built workload of golden/model_hand.txt,
and deliberately broken copies of oracle/model.py (each must fail a pin): the K and
V weight pairs swapped, layer 1 composed, the cross-decoder layers reading layer
L/2 - 1, the query-head slice of a group off by one, a self-decoder layer reading
the shared cache, prefill rows seeing one position too many."""
import importlib.util
import os
import sys

import pytest

import oracle
from oracle import model
from model_pins import MODEL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "model.py")


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", MODEL_PINS, ids=lambda f: f.__name__)
def test_model_pin(orc, pin):
    pin(orc, model)


def _in_function(text, fn, old, new):
    """Replace ``old`` (once) inside the body of function ``fn`` of model.py."""
    start = text.index(f"\ndef {fn}(")
    end = text.find("\ndef ", start + 1)
    end = len(text) if end < 0 else end
    body = text[start:end]
    assert body.count(old) >= 1, f"anchor {old!r} not in {fn}"
    return text[:start] + body.replace(old, new, 1) + text[end:]


MUTANTS = {
    "swap_kv_alpha_pairs": ("composed_seq", "(a[0], a[1]) if which == \"K\" else (a[2], a[3])",
                            "(a[2], a[3]) if which == \"K\" else (a[0], a[1])"),
    "alpha_within_pair_swapped": ("composed_seq", "a1, a2 = (a[0], a[1])", "a2, a1 = (a[0], a[1])"),
    "layer1_composed": ("composed_seq", "if layer == 1:", "if layer == 0:"),
    "shared_layer_minus_one": ("decode_group", "composed_seq(orc, w, w.shared_layer, \"K\"",
                               "composed_seq(orc, w, w.shared_layer - 1, \"K\""),
    "shared_layer_minus_one_both": ("decode_group", "K = composed_seq(orc, w, w.shared_layer, \"K\", b, g)\n"
                                                    "        V = composed_seq(orc, w, w.shared_layer, \"V\", b, g)",
                                    "K = composed_seq(orc, w, w.shared_layer - 1, \"K\", b, g)\n"
                                    "        V = composed_seq(orc, w, w.shared_layer - 1, \"V\", b, g)"),
    "group_slice_off_by_one": ("decode_group", "[g * w.group:(g + 1) * w.group]",
                               "[g * w.group + 1:(g + 1) * w.group + 1]"),
    "group_slice_by_kv_head": ("decode_group", "[g * w.group:(g + 1) * w.group]", "[g:g + w.group]"),
    "self_reads_shared": ("decode_self_group", "K = composed_seq(orc, w, layer, \"K\", b, g)",
                          "K = composed_seq(orc, w, w.shared_layer, \"K\", b, g)"),
    "self_query_from_cross_layer": ("decode_self_group", "q = query(w, layer, b)", "q = query(w, layer + 2, b)"),
    "decoded_token_dropped": ("raw_seq", "return np.concatenate([pre, new], axis=0)",
                              "return np.concatenate([pre, pre[-1:]], axis=0)"),
    "prefill_sees_next_position": ("prefill_self_rows", "p0=int(t)", "p0=int(t) + 1"),
    "prefill_queries_reversed": ("prefill_queries", "block[rows - lo]", "block[::-1][rows - lo]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_model_mutant_is_caught(orc, name, tmp_path):
    fn, old, new = MUTANTS[name]
    with open(SRC) as f:
        text = f.read()
    text = _in_function(text, fn, old, new).replace("from . import", "from oracle import")
    path = tmp_path / f"model_{name}.py"
    path.write_text(text)
    spec = importlib.util.spec_from_file_location(f"_model_mutant_{name}", path)
    mdl = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mdl)
    failed = []
    for pin in MODEL_PINS:
        try:
            pin(orc, mdl)
        except (AssertionError, KeyError, IndexError, ValueError) as e:
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"model mutant {name} passed every pin"
