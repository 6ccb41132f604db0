"""Every plausible slip in the oracle must be caught by at least one pin.

Each mutant is a textual edit of oracle.c (a dropped term, a wrong sign, a
swapped index or operand, a missing factor), compiled on the CPU into a
temporary library; the pin suite must reject every one of them.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "swap_alpha": ("a1 * load(x1, dtype, j) + a2 * load(xi, dtype, j)",
                   "a2 * load(x1, dtype, j) + a1 * load(xi, dtype, j)"),
    "drop_lambda": ("out[j] = lam * inner;", "out[j] = inner;"),
    "drop_k1_term": ("a1 * load(x1, dtype, j) + a2", "0.0 * load(x1, dtype, j) + a2"),
    "bf16_low_half": ("(uint32_t)((const uint16_t*)base)[i] << 16", "(uint32_t)((const uint16_t*)base)[i] << 15"),
    "round_truncate": ("double r = nearbyint(ldexp(m, bits));", "double r = floor(ldexp(m, bits));"),
    "round_half_up": ("double r = nearbyint(ldexp(m, bits));", "double r = floor(ldexp(m, bits) + 0.5);"),
    "transposed_K": ("for (int c = 0; c < d; ++c) dot += qh[c] * load(K, dtype, t * d + c);\n            scores[t] = scale * dot;",
                     "for (int c = 0; c < d; ++c) dot += qh[c] * load(K, dtype, c * len + t);\n            scores[t] = scale * dot;"),
    "no_scale": ("scores[t] = scale * dot;", "scores[t] = dot;"),
    "softmax_sign": ("Z += exp(scores[t] - mx);", "Z += exp(mx - scores[t]);"),
    "unnormalised": ("double p = exp(scores[t] - mx) / Z;", "double p = exp(scores[t] - mx);"),
    "value_from_key": ("oh[c] += p * load(V, dtype, t * d + c);\n        }\n    }\n}",
                       "oh[c] += p * load(K, dtype, t * d + c);\n        }\n    }\n}"),
    "first_token_skipped": ("for (int64_t t = 0; t < len; ++t) Z += exp(scores[t] - mx);",
                            "for (int64_t t = 1; t < len; ++t) Z += exp(scores[t] - mx);"),
    "combine_no_rescale": ("double w = exp(m[s * G + h] - M);", "double w = 1.0;"),
    "combine_no_divide": ("for (int c = 0; c < d; ++c) oh[c] /= L;", ""),
    "partial_wrong_max": ("if (s > mx) mx = s;", "if (s < mx) mx = s;"),
    "head_stride": ("const double* qh = q + (int64_t)h * d;\n        double* oh", "const double* qh = q;\n        double* oh"),
    "causal_excludes_self": ("const int64_t visible = p0 + j + 1;", "const int64_t visible = p0 + j;"),
    "causal_ignores_offset": ("const int64_t visible = p0 + j + 1;", "const int64_t visible = j + 1;"),
    "causal_whole_chunk": ("const int64_t visible = p0 + j + 1;", "const int64_t visible = p0 + n;"),
    "causal_first_query": ("orc_attention(q + j * d, K, V", "orc_attention(q, K, V"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        text = f.read()
    assert text.count(old) == 1, f"mutation anchor for {name} not unique in oracle.c"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    so = oracle.build(force=True, src=str(src), out=str(tmp_path / "mutant.so"))
    orc = oracle.Oracle(oracle.load(so))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
