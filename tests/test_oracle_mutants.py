"""The pins catch plausible mistakes in the oracle.

Each case plants one mistake (a dropped term, a wrong sign, a wrong index,
a transposed bit) in a copy of oracle/onebit_oracle.c, builds it with gcc
into a temporary directory, and requires at least one pin of
tests/oracle_pins.py to fail on it.  Mistakes are only ever planted in the
oracle, on the CPU; none of them reads out of bounds.
"""
import os
import subprocess

import pytest

import oracle
import oracle_pins

# (name, text in the oracle, replacement)
MUTANTS = [
    ("warmup_drops_bias_correction_m", "const float mhat = m[i] / bc1;", "const float mhat = m[i];"),
    ("warmup_eps_inside_sqrt",
     "const float root = sqrtf(vhat);\n    const float denom = root + eps;",
     "const float root = sqrtf(vhat + eps);\n    const float denom = root;"),
    ("warmup_sums_instead_of_averaging", "const float gbar = acc / wf;", "const float gbar = acc;"),
    ("warmup_variance_not_squared", "const float gsq = gbar * gbar;", "const float gsq = gbar;"),
    ("warmup_update_wrong_sign", "p[i] = p[i] - delta;\n    }\n}\n\n/* [1BA, Abstract; Proposed",
     "p[i] = p[i] + delta;\n    }\n}\n\n/* [1BA, Abstract; Proposed"),
    ("freeze_drops_bias_correction",
     "const float vhat = v[i] / bc2;\n        const float root = sqrtf(vhat);\n        d[i]",
     "const float vhat = v[i];\n        const float root = sqrtf(vhat);\n        d[i]"),
    ("sign_of_zero_is_minus", "return x >= 0.0f ? 1 : 0;", "return x > 0.0f ? 1 : 0;"),
    ("scale_divides_by_n", "return (float)sqrt(sum_sq / (double)count);",
     "return (float)(sqrt(sum_sq) / (double)count);"),
    ("scale_is_mean_square", "return (float)sqrt(sum_sq / (double)count);",
     "return (float)(sum_sq / (double)count);"),
    ("worker_error_wrong_sign", "e[i] = x[i] - signed_scale(", "e[i] = x[i] + signed_scale("),
    ("momentum_drops_old_m", "const float m_old = beta1 * m[i];\n        const float m_new = c1 * g[i];",
     "const float m_old = 0.0f * m[i];\n        const float m_new = c1 * g[i];"),
    ("momentum_drops_gradient",
     "const float m_old = beta1 * m[i];\n        const float m_new = c1 * g[i];",
     "const float m_old = beta1 * m[i];\n        const float m_new = c1 * 0.0f * g[i];"),
    ("worker_forgets_error", "x[i] = m_w + e[i];", "x[i] = m_w;"),
    ("server_does_not_average", "const float avg = acc / wf;", "const float avg = acc;"),
    ("server_forgets_error", "y[i - b] = avg + e_s[i];", "y[i - b] = avg;"),
    ("server_uses_worker0_scale", "signed_scale(get_bit(bits[w], i), s[w])",
     "signed_scale(get_bit(bits[w], i), s[0])"),
    ("server_reads_neighbour_bit", "signed_scale(get_bit(bits[w], i), s[w])",
     "signed_scale(get_bit(bits[w], i ^ 1), s[w])"),
    ("server_error_uses_worker0_scale",
     "e_s[i] = y[i - b] - signed_scale(sign_bit(y[i - b]), sj);",
     "e_s[i] = y[i - b] - signed_scale(sign_bit(y[i - b]), s[0]);"),
    ("server_error_wrong_sign", "e_s[i] = y[i - b] - signed_scale(", "e_s[i] = y[i - b] + signed_scale("),
    ("chunks_not_word_group_aligned", "const int64_t cw = ((per + 3) / 4) * 4;",
     "const int64_t cw = per;"),
    ("apply_wrong_sign", "p[i] = p[i] - delta;\n        m[i] = m_hat;",
     "p[i] = p[i] + delta;\n        m[i] = m_hat;"),
    ("apply_keeps_old_momentum", "        m[i] = m_hat;\n", "        (void)m;\n"),
    ("apply_uses_chunk0_scale", "orc_apply_chunk(n, W, j, lr, sbits, s_srv[j], d, p, m);",
     "orc_apply_chunk(n, W, j, lr, sbits, s_srv[0], d, p, m);"),
    ("apply_multiplies_by_d", "const float ratio = m_hat / d[i];", "const float ratio = m_hat * d[i];"),
    ("packing_bit_order_reversed", "words[i >> 5] |= (uint32_t)1u << (i & 31);",
     "words[i >> 5] |= (uint32_t)1u << (31 - (i & 31));"),
    ("server_packing_bit_order_reversed", "sbits[i >> 5] |= (uint32_t)1u << (i & 31);",
     "sbits[i >> 5] |= (uint32_t)1u << (31 - (i & 31));"),
    ("server_empty_chunk_clears_a_word", "    if (e > b)  /* an empty chunk owns no word, not even the tensor's last */\n",
     "    if (1)\n"),
    ("freeze_eps_inside_sqrt",
     "const float root = sqrtf(vhat);\n        d[i] = root + eps;",
     "const float root = sqrtf(vhat + eps);\n        d[i] = root;"),
    ("scale_uses_n_minus_1", "return (float)sqrt(sum_sq / (double)count);",
     "return (float)sqrt(sum_sq / (double)(count > 1 ? count - 1 : 1));"),
    ("worker_momentum_constants_swapped",
     "const float m_old = beta1 * m[i];\n        const float m_new = c1 * g[i];",
     "const float m_old = c1 * m[i];\n        const float m_new = beta1 * g[i];"),
    ("warmup_variance_uses_beta1", "const float v_old = beta2 * v[i];", "const float v_old = beta1 * v[i];"),
    ("chunk_words_rounded_down", "const int64_t per = (nw + W - 1) / W;", "const int64_t per = nw / W;"),
    # 1-bit LAMB
    ("lamb_ratio_inverted", "return (float)sqrt(p_sq / u_sq);", "return (float)sqrt(u_sq / p_sq);"),
    ("lamb_ratio_without_root", "return (float)sqrt(p_sq / u_sq);", "return (float)(p_sq / u_sq);"),
    ("lamb_zero_norm_gives_zero_rate", "    return 1.0f;\n}", "    return 0.0f;\n}"),
    ("lamb_warmup_ignores_ratio", "const float lr_t = lr * ratio;\n    for", "const float lr_t = lr;\n    for"),
    ("lamb_warmup_ratio_of_momentum", "orc_sum_squares(n, r));", "orc_sum_squares(n, m));"),
    ("lamb_warmup_ratio_of_variance", "trust_ratio(orc_sum_squares(n, p), orc_sum_squares(n, r))",
     "trust_ratio(orc_sum_squares(n, v), orc_sum_squares(n, r))"),
    ("lamb_compressed_ratio_of_d", "return trust_ratio(orc_sum_squares(n, p), u_sq);",
     "return trust_ratio(orc_sum_squares(n, d), u_sq);"),
    ("lamb_compressed_ratio_ignores_d", "/ (double)d[i];", "/ 1.0;"),
    ("lamb_compressed_ratio_chunk0_scale", "signed_scale(get_bit(sbits, i), s_srv[j]) / (double)d[i]",
     "signed_scale(get_bit(sbits, i), s_srv[0]) / (double)d[i]"),
    ("lamb_apply_ignores_ratio", "const float lr_t = lr * ratio;\n    orc_apply_chunk",
     "const float lr_t = lr + 0.0f * ratio;\n    orc_apply_chunk"),
]

MUTANT_CFLAGS = [f for f in oracle.CFLAGS if f != "-Werror"]


@pytest.fixture(scope="module")
def source():
    with open(oracle.SOURCE) as f:
        return f.read()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new, source, tmp_path):
    assert source.count(old) == 1, f"mutation site for {name} not unique in the oracle"
    src = tmp_path / f"{name}.c"
    src.write_text(source.replace(old, new))
    lib = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", *MUTANT_CFLAGS, "-o", str(lib), str(src), "-lm"])
    mutant = oracle.Oracle(str(lib))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name}"


# Mistakes in the runner's frozen-ratio bookkeeping (the 1-bit LAMB
# reading whose ratios are kept at the freeze): planted by wrapping
# OracleRun's methods; pin_lamb_frozen_ratio_run must fail on each.
def _recompute_after_freeze(run_cls):
    freeze = run_cls.freeze

    def patched(self):
        freeze(self)
        self.lamb_frozen = False          # the ratios recomputed after all
    return {"freeze": patched}


def _keep_first_warmup_ratio(run_cls):
    warmup_step, freeze = run_cls.warmup_step, run_cls.freeze

    def warm(self, grads):
        warmup_step(self, grads)
        if self.t_warmup == 1:
            self._first_ratio = self.ratio.copy()

    def frz(self):
        freeze(self)
        if self.lamb_frozen:
            self.frozen_ratio = self._first_ratio.copy()   # the first step's, not the last
    return {"warmup_step": warm, "freeze": frz}


@pytest.mark.parametrize("plant", [_recompute_after_freeze, _keep_first_warmup_ratio],
                         ids=["recomputed_after_freeze", "first_warmup_ratio_kept"])
def test_frozen_ratio_pin_catches_runner_mistakes(plant, monkeypatch):
    for name, fn in plant(oracle.OracleRun).items():
        monkeypatch.setattr(oracle.OracleRun, name, fn)
    with pytest.raises(AssertionError):
        oracle_pins.pin_lamb_frozen_ratio_run(oracle.default())
