"""Planted mistakes in a copy of the oracle must each be caught by a pin.

Every mutant is one plausible slip (a sign, a dropped term, a wrong index, a
transposed operand, a wrong rounding); the copy is compiled on the CPU and the
pins of ``oracle_pins`` are run against it. A mutant that passes every pin
means the pins leave that part of the oracle unchecked.
"""
import os
import shutil

import pytest

import oracle
from oracle import build as obuild
import oracle_pins

MUTANTS = {
    "lse_sign": ("return m + log(s);", "return m - log(s);"),
    "lse_accepts_negative_sum": ("!(s > 0.0)", "!(s != 0.0)"),
    "lse_accepts_inf_max": ("if (!isfinite(m) || !isfinite(s)", "if (isnan(m) || !isfinite(s)"),
    "combine_no_max_shift": ("sum += exp(lse[r] - M);", "sum += exp(lse[r]);"),
    "combine_unnormalised": ("double w = exp(lse[r] - L);", "double w = exp(lse[r] - M);"),
    "combine_rank_index": ("out[d] += w * o[r * D + d];", "out[d] += w * o[d];"),
    "combine_invalid_not_skipped": ("if (!(lse[r] > -INFINITY))\n            continue;", ""),
    "combine_max_is_min": ("if (lse[r] > M)\n                M = lse[r];",
                           "if (lse[r] < M || M == -INFINITY)\n                M = lse[r];"),
    "pack_chunk_index": ("j = h / Hc;", "j = h % W;"),
    "pack_slot_transposed": ("slot = t * Hc + (h % Hc);", "slot = (h % Hc) * T + t;"),
    "pack_token_chunks_interleaved": ("j = t / Tc;\n                    slot = (t % Tc) * H + h;",
                                      "j = t % W;\n                    slot = (t / W) * H + h;"),
    "pack_token_slot_transposed": ("slot = (t % Tc) * H + h;", "slot = h * Tc + (t % Tc);"),
    "permute_identity": ("memcpy(recv + ((int64_t)j * W + r) * block_bytes",
                         "memcpy(recv + ((int64_t)r * W + j) * block_bytes"),
    "seq2head_interleaved": ("* S + (int64_t)r * S_l + s) * Hc + hc;",
                             "* S + s * W + r) * Hc + hc;"),
    "head2seq_chunk": ("* S + (int64_t)j * S_l + s) * Hc + hc;", "* S + s * W + j) * Hc + hc;"),
    "fp16_exponent": ("ex - 25", "ex - 24"),
    "round_truncates": ("double q = nearbyint(a / spacing);", "double q = floor(a / spacing);"),
    "fused_chunk_offset": ("int64_t j = h / Hc, hc = h % Hc;", "int64_t j = h % W, hc = h / W;"),
    "legacy_lse_index": ("pkt_lse[dst_row] = lse[r * sl_r + t * sl_t + h * sl_h];",
                         "pkt_lse[dst_row] = lse[r * sl_r + h * sl_t + t * sl_h];"),
}


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_mutants")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, mutant_dir):
    old, new = MUTANTS[name]
    src = open(obuild.SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    d = mutant_dir / name
    d.mkdir()
    path = str(d / "m.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new, 1))
    lib = obuild.compile_oracle(path, str(d / "libm.so"))
    mut = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mut)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
    shutil.rmtree(str(d), ignore_errors=True)
