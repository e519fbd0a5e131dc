"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the pins
catch each one: a pin set that a dropped term, a wrong sign or index, or a swapped operand
slips through would not be pinning anything."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle
from tests import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "pspec_oracle.c")

# (name, text in pspec_oracle.c, replacement)
MUTANTS = [
    ("residual_abs_not_max", "r[t] = diff > 0.0 ? diff : 0.0;", "r[t] = diff > 0.0 ? diff : -diff;"),
    ("ratio_inverted", "double ratio = pk[k] / qk[k];", "double ratio = qk[k] / pk[k];"),
    ("accept_le", "accept = (double)u[k] < ratio;", "accept = (double)u[k] <= ratio + 1e-3;"),
    ("resample_wrong_row", "long long toff = ((long long)i * (K + 1) + a) * ld;",
     "long long toff = ((long long)i * (K + 1) + (a < K ? a + 1 : a)) * ld;"),
    ("residual_swapped", "double diff = row_prob(target_logits, dtype, toff, t, lse_t[a]) -\n"
     "                              row_prob(draft_logits, dtype, qoff, t, lse_q[a]);",
     "double diff = row_prob(draft_logits, dtype, qoff, t, lse_q[a]) -\n"
     "                              row_prob(target_logits, dtype, toff, t, lse_t[a]);"),
    ("inverse_cdf_ge", "cum += r[t];\n            if (cum > thr) { tok = t; break; }",
     "cum += r[t];\n            if (cum >= thr + 0.01) { tok = t; break; }"),
    ("bonus_from_row_k_minus_1", "long long toff = ((long long)i * (K + 1) + a) * ld;",
     "long long toff = ((long long)i * (K + 1) + (a == K ? K - 1 : a)) * ld;"),
    ("lse_dropped_shift", "for (int t = 0; t < V; ++t) s += exp(logit_at(base, dtype, off + t) - m);\n    return m + log(s);",
     "for (int t = 0; t < V; ++t) s += exp(logit_at(base, dtype, off + t) - m);\n    return log(s);"),
    ("argmax_last_tie", "if (x > bv) { bv = x; best = t; }", "if (x >= bv) { bv = x; best = t; }"),
    ("greedy_bonus_row_off", "out[a] = amax[a];", "out[a] = amax[a > 0 ? a - 1 : 0];"),
    ("bf16_wrong_half", "uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;",
     "uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 15;"),
    ("eagle_shift_missing", "tok = verify_tokens[s + j + 1];", "tok = verify_tokens[s + j];"),
    ("mask_pos_off", "pos = ntp_pos + m;", "pos = ntp_pos + m - 1;"),
    ("rejected_slot_kept", "slot = -1;                /* PADDING_SLOT_ID */",
     "slot = kv_slot(block_table, max_blocks, block_size, i, pos, &e);"),
    ("ntp_hidden_off", "src = s + j;\n                kind = ORACLE_ROW_NTP;",
     "src = s + j - 1;\n                kind = ORACLE_ROW_NTP;"),
    ("slot_formula_swapped", "return (long long)id * block_size + pos % block_size;",
     "return (long long)id * block_size + pos / block_size;"),
    ("sample_cdf_ge", "if (cum > thr) { tok = t; break; }\n            }\n            if (tok < 0) {\n                tok = last_pos >= 0 ? last_pos : 0;\n                flag = 2;\n            } else if (thr - prev < tie_eps * Z",
     "if (cum + 0.05 > thr) { tok = t; break; }\n            }\n            if (tok < 0) {\n                tok = last_pos >= 0 ? last_pos : 0;\n                flag = 2;\n            } else if (thr - prev < tie_eps * Z"),
    ("sample_greedy_last_tie", "            tok = row_argmax(logits, dtype, off, V);\n        } else {",
     "            tok = row_argmax(logits, dtype, off, V) + (V > 1);\n        } else {"),
    ("offsets_without_masks", "off += (qsl_in[i + 1] - qsl_in[i]) + K - 1;", "off += (qsl_in[i + 1] - qsl_in[i]) + K;"),
    ("k_len_draw_column_K", "double thr = (double)u[Ki] * Z;", "double thr = (double)u[K] * Z;"),
    ("k_len_accept_loop_K", "int a = Ki;\n        for (int k = 0; k < Ki; ++k) {",
     "int a = K;\n        for (int k = 0; k < K; ++k) {"),
    ("k_len_greedy_ignored", "while (a < Ki) {", "while (a < K) {"),
    ("k_len_build_survivors", "int c = L - Ki + a;", "int c = L - K + a;"),
]


_CHILD = r"""
import sys
sys.path[:0] = [{root!r}]
import oracle
from tests import oracle_pins as P
lib = oracle.OracleLib({lib!r})
for pin in P.ALL_PINS:                  # cheap pins first; the first failure is enough
    try:
        pin(lib)
    except Exception:  # noqa: BLE001
        print("CAUGHT", pin.__name__)
        break
else:
    print("MISSED")
"""


def _run_mutant(tmpdir, name, old, new):
    src = open(SRC).read()
    if src.count(old) != 1:
        return f"mutation site for {name} not found exactly once"
    d = os.path.join(tmpdir, name)
    os.makedirs(d, exist_ok=True)
    mut = os.path.join(d, "pspec_oracle.c")
    with open(mut, "w") as f:
        f.write(src.replace(old, new))
    so = oracle.build(force=True, src=mut, out=os.path.join(d, "lib.so"))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _CHILD.format(root=root, lib=so)],
                         capture_output=True, text=True, timeout=600)
    if res.returncode != 0:
        return "caught (crashed)"                # a memory-corrupting mutant is caught too
    return res.stdout.strip().splitlines()[-1] if res.stdout.strip() else "no output"


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """Compile every mutant and run the pins on each in its own child process, in parallel:
    a crash counts as caught and cannot take the test session down."""
    tmpdir = str(tmp_path_factory.mktemp("mutants"))
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        futs = {m[0]: ex.submit(_run_mutant, tmpdir, *m) for m in MUTANTS}
        return {k: f.result() for k, f in futs.items()}


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_pins_catch_mutant(mutant_results, name):
    assert mutant_results[name].startswith(("CAUGHT", "caught")), \
        f"mutant {name}: {mutant_results[name]}"
