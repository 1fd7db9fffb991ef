"""The oracle's pins catch plausible mistakes.

Each case patches one line of a *copy* of the oracle's C source (a dropped term, a wrong
sign, a wrong index, a transposed operand ...), compiles the copy into a temporary
library on the CPU, and runs the pins of ``test_oracle.py`` against it: at least one pin
must fail.  The oracle source itself is never modified.
"""
import os
import tempfile

import pytest

import oracle
import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "pkv_oracle.c")

MUTANTS = {
    "gqa_head_mapping": ("const int64_t kvh = h / G;", "const int64_t kvh = h % Hkv;"),
    "token_offset": ("const int64_t offset = t % bs;", "const int64_t offset = (t + 1) % bs;"),
    "logical_block": ("const int64_t logical = t / bs;", "const int64_t logical = t / bs / 2;"),
    "softmax_sign": ("exp(s[t] - smax)", "exp(smax - s[t])"),
    "dropped_scale": ("s[t] = scale * acc;", "s[t] = acc;"),
    "dropped_normalisation": ("out_row[d] /= wsum;", "out_row[d] /= 1.0;"),
    "dropped_dot_term": ("for (d = 0; d < D; ++d) acc +=", "for (d = 1; d < D; ++d) acc +="),
    "q_head_index": ("(b * Hq + h) * D, k_cache", "(b * Hq + kvh) * D, k_cache"),
    "prefill_causal_bound": ("seq_lens[b] - Q + i + 1;", "seq_lens[b] - Q + i;"),
    "prefill_kv_head": ("const int64_t kv_head = h / (Hq / Hkv);", "const int64_t kv_head = h % Hkv;"),
    "prefill_q_row": ("attend_row(out + r * D, q, r * D,", "attend_row(out + r * D, q, row * D,"),
    "k_for_v_operand": ("out_row[d] += w * Vc[t * D + d];", "out_row[d] += w * Kc[t * D + d];"),
    "write_offset": ("const int64_t offset = s % bs;", "const int64_t offset = (s + 1) % bs;"),
    "write_block": ("const int64_t block = s / bs;", "const int64_t block = s / (bs + 1);"),
    "write_skips_v": (
        "memcpy((char *)v_cache + dst * es, (const char *)v + src * es, (size_t)es);",
        "memcpy((char *)v_cache + dst * es, (const char *)k + src * es, (size_t)es);"),
    "copy_half_block": ("for (int64_t byte = 0; byte < block_bytes; ++byte)",
                        "for (int64_t byte = 0; byte < block_bytes / 2; ++byte)"),
    "copy_v_from_k": (
        "((char *)v_cache)[dst * block_bytes + byte] = ((const char *)v_cache)[src * block_bytes + byte];",
        "((char *)v_cache)[dst * block_bytes + byte] = ((const char *)k_cache)[src * block_bytes + byte];"),
    "bf16_widening": ("((uint32_t)h) << 16", "((uint32_t)h) << 15"),
    "floor_block_count": ("if (n * block_size < token_count) n += 1;", ""),
    "no_max_guard_in_range": ("if (L > max_blocks * bs) return -2;", ""),
}

PIN_NAMES = [n for n in dir(pins) if n.startswith("test_")]


@pytest.fixture(scope="module")
def workdir():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, workdir):
    before, after = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(before) == 1, f"pattern for {name} must occur exactly once"
    path = os.path.join(workdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(text.replace(before, after))
    lib = oracle.build(force=True, src=path, out=os.path.join(workdir, f"lib{name}.so"))
    mutant = oracle.Oracle(lib)
    failed = []
    for pin in PIN_NAMES:
        try:
            getattr(pins, pin)(o=mutant)
        except (Exception, pytest.fail.Exception) as e:  # assertion, error or pytest failure
            failed.append((pin, type(e).__name__))
            break
    assert failed, f"no pin caught mutant {name}"
