"""The pins can tell a broken oracle from the real one (CPU only).

Each case copies the oracle's sources, plants one plausible mistake in the copy
(a wrong recurrence, a dropped sign, a wrong octant rule, a wrong series
coefficient, the vocabulary chunk's offset forgotten in the noise channel, a
reward that runs past its sequence, a wrong attention score scale), builds
it, and runs the pin meant to catch that kind of mistake against the broken
build: the pin must fail.  The committed oracle is untouched; only the copy is
broken."""
import importlib
import os
import shutil

import numpy as np
import pytest

import oracle

import suffix_autograd as SA
import test_noise_spec as NS
import test_oracle_pins as OP

oracle_build = importlib.import_module("oracle.build")
HERE = os.path.dirname(os.path.abspath(oracle.__file__))


def _clean_losses_match_autograd(orc):
    """Clean per-token losses of the toy suffix against float64 torch (the
    config-2 pin's first step)."""
    p = SA.tiny_problem()
    clean = orc.toy_suffix_losses(p["X"], p["W"], p["off"], p["Wq"], p["Wk"], p["Wv"], p["Wo"], p["Wout"], p["y"],
                                  0, 5, 0.01, [0], with_noise=False)[0]
    np.testing.assert_allclose(SA.clean_losses(p), clean, rtol=1e-12)


MUTANTS = [
    ("scan recurrence discounts twice", "estimator.c",
     "acc = (double)ci[t] + gamma * acc;", "acc = (double)ci[t] + gamma * gamma * acc;",
     lambda orc: OP.test_scan_recurrence_equals_brute_force(orc, 0.9)),
    ("error estimate without its minus sign", "estimator.c",
     "const double scale = -1.0 / ((double)K_total * sigma);", "const double scale = 1.0 / ((double)K_total * sigma);",
     OP.test_estimate_single_draw_closed_form),
    ("reward runs past the end of its sequence", "estimator.c",
     "for (int s = seq_offsets[q + 1] - 1; s >= t; --s)", "for (int s = T - 1; s >= t; --s)",
     OP.test_estimate_reward_path_and_draw_split),
    ("sine and cosine swapped in the wrong octants", "noise.c",
     "uint32_t swap = ((o + 1u) >> 1) & 1u;", "uint32_t swap = (o >> 1) & 1u;",
     NS.test_box_muller_matches_exact_transform),
    ("atanh series coefficient 1/7 typed as 1/5", "noise.c",
     "static const float LN_C7  = 0x1.24924ap-3f;", "static const float LN_C7  = 0x1.99999ap-3f;",
     NS.test_ln_exhaustive_within_2ulp),
    ("head noise channel forgets the chunk offset", "head.c",
     "(uint32_t)(v0 + j), 0);", "(uint32_t)j, 0);",
     OP.test_head_costs_brute_force_mpmath),
    ("attention scores not scaled by 1/sqrt(dh)", "suffix.c",
     "sc *= inv_sqrt_dh;", "sc *= 1.0;",
     _clean_losses_match_autograd),
]


@pytest.fixture(scope="module")
def real_oracle():
    return oracle.lib()


@pytest.mark.parametrize("name,src,old,new,pin", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pin_catches_planted_mistake(real_oracle, tmp_path, name, src, old, new, pin):
    for f in os.listdir(HERE):
        if f.endswith((".c", ".h")):
            shutil.copy(os.path.join(HERE, f), tmp_path / f)
    text = (tmp_path / src).read_text()
    assert text.count(old) == 1, f"mutation site not found once in {src}: {old}"
    (tmp_path / src).write_text(text.replace(old, new))
    broken = oracle.load(oracle_build.compile_sources(str(tmp_path), str(tmp_path / "liboracle_broken.so")))
    pin(oracle)                                   # the pin passes on the real oracle
    oracle._lib = broken
    try:
        with pytest.raises(AssertionError):
            pin(oracle)                           # and fails on the broken copy
    finally:
        oracle._lib = real_oracle
