"""The C-ABI library loads, exports every symbol include/dust.h declares, and
rejects invalid calls on the host (CPU only: no call here reaches a kernel)."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from activation_perturbation_es_b200 import build as B
from activation_perturbation_es_b200 import dust

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return dust.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "dust.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dust_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert len(names) >= 18
    for n in names:
        assert hasattr(L, n), n
    # the binding covers the whole ABI
    assert set(names) == set(dust._SIGS)


def test_no_oracle_linkage():
    """The product library neither links nor names the CPU oracle."""
    data = open(B.LIB, "rb").read()
    assert b"orc_" not in data and b"liboracle" not in data


def test_status_strings_and_version(L):
    assert L.dust_abi_version() == 2
    for s, name in dust.STATUS.items():
        assert L.dust_status_string(s).decode() == name


def test_check_offsets(L):
    dust.check_offsets([0, 3, 3, 10], 10)
    for bad, T in [([1, 3, 10], 10), ([0, 5, 4, 10], 10), ([0, 5, 9], 10)]:
        with pytest.raises(dust.DustError) as e:
            dust.check_offsets(bad, T)
        assert e.value.status == 1


NZ = dust.Noise(0, 0, 0, 4, 4, 0.01)
GOOD = 0x10000   # aligned fake device address: never dereferenced (validation fails first)


def status(call):
    return int(call)


def test_invalid_sizes_rejected_on_host(L):
    st = None
    assert status(L.dust_reward_scan(GOOD, GOOD, 0, 16, GOOD, 1, 0.5, st)) == 1          # K = 0
    assert status(L.dust_reward_scan(GOOD, GOOD, 4, 0, GOOD, 1, 0.5, st)) == 1           # T = 0
    assert status(L.dust_reward_scan(GOOD, GOOD, 4, 16, GOOD, 1, 1.5, st)) == 1          # gamma > 1
    assert status(L.dust_reward_scan(GOOD, GOOD, 4, 16, GOOD, 0, 0.5, st)) == 1          # n_seq = 0
    assert status(L.dust_reward_scan(GOOD, None, 4, 16, GOOD, 1, 0.5, st)) == 1          # NULL output
    nz0 = dust.Noise(0, 0, 0, 0, 4, 0.01).c()                                            # draw_count = 0
    assert status(L.dust_layer_estimate(GOOD, 1, 16, 8, GOOD, 1, 0.0, nz0, GOOD, None, 0, None, 0, st)) == 1
    bad_sigma = dust.Noise(0, 0, 0, 4, 4, 0.0).c()
    assert status(L.dust_layer_estimate(GOOD, 1, 16, 8, GOOD, 1, 0.0, bad_sigma, GOOD, None, 0, None, 0, st)) == 1
    wrap = dust.Noise(0, 0, 2**32 - 2, 4, 4, 0.01).c()                                  # draw index overflow
    assert status(L.dust_layer_estimate(GOOD, 1, 16, 8, GOOD, 1, 0.0, wrap, GOOD, None, 0, None, 0, st)) == 1
    assert status(L.dust_layer_estimate(GOOD, 1, 16, 8, GOOD, 1, 0.0, NZ.c(), None, None, 0, None, 0, st)) == 1
    # head: Vc must divide V and be supported
    assert status(L.dust_head_step(None, None, 0, GOOD, GOOD, 16, 0, 1000, 300, 0, 3, NZ.c(), None, GOOD, None,
                                   None, 0, GOOD, 1 << 20, st)) == 1
    assert status(L.dust_head_step(None, None, 0, GOOD, GOOD, 16, 0, 960, 96, 0, 10, NZ.c(), None, GOOD, None, None,
                                   0, GOOD, 1 << 20, st)) == 2
    # Z missing and no X/W to recompute it
    assert status(L.dust_head_step(None, None, 0, None, GOOD, 16, 8, 512, 128, 0, 4, NZ.c(), None, GOOD, None, None,
                                   0, GOOD, 1 << 20, st)) == 1
    # chunk ranges outside the V/Vc chunks
    for cb, cc in ((0, 0), (-1, 2), (3, 2), (4, 1)):
        assert status(L.dust_head_step(None, None, 0, GOOD, GOOD, 16, 0, 512, 128, cb, cc, NZ.c(), None, GOOD,
                                       None, None, 0, GOOD, 1 << 20, st)) == 1
    assert "chunk range" in L.dust_last_error().decode()
    # token_begin past 2^31
    far = dust.Noise(0, 0, 0, 4, 4, 0.01, 2**31).c()
    assert status(L.dust_layer_estimate(GOOD, 1, 16, 8, GOOD, 1, 0.0, far, GOOD, None, 0, None, 0, st)) == 1
    # weight_grad: unknown dtype, zero sizes
    assert status(L.dust_weight_grad(GOOD, 7, GOOD, 0, 16, 8, 8, GOOD, 0, GOOD, 1 << 20, st)) == 1
    assert status(L.dust_weight_grad(GOOD, 0, GOOD, 7, 16, 8, 8, GOOD, 0, GOOD, 1 << 20, st)) == 1
    assert status(L.dust_weight_grad(GOOD, 0, GOOD, 0, 0, 8, 8, GOOD, 0, GOOD, 1 << 20, st)) == 1
    assert "must" in L.dust_last_error().decode()
    # noise sum: empty shapes, no draws, token range past 2^31
    assert status(L.dust_noise_sum(NZ.c(), 0, 8, GOOD, st)) == 1
    assert status(L.dust_noise_sum(NZ.c(), 16, 0, GOOD, st)) == 1
    assert status(L.dust_noise_sum(nz0, 16, 8, GOOD, st)) == 1
    assert status(L.dust_noise_sum(far, 16, 8, GOOD, st)) == 1
    assert status(L.dust_noise_sum(NZ.c(), 16, 8, None, st)) == 1


def test_misaligned_pointers_rejected_on_host(L):
    st = None
    assert status(L.dust_reward_scan(GOOD + 4, GOOD, 4, 16, GOOD, 1, 0.5, st)) == 3
    assert status(L.dust_reward_scan(GOOD, GOOD + 8, 4, 16, GOOD, 1, 0.5, st)) == 3
    assert status(L.dust_layer_estimate(GOOD, 1, 16, 8, GOOD, 1, 0.0, NZ.c(), GOOD + 2, None, 0, None, 0, st)) == 3
    assert status(L.dust_weight_grad(GOOD, 0, GOOD + 4, 1, 16, 8, 8, GOOD, 0, GOOD, 1 << 20, st)) == 3
    assert status(L.dust_noise_sum(NZ.c(), 16, 8, GOOD + 4, st)) == 3
    assert "aligned" in L.dust_last_error().decode()


def test_workspace_too_small_rejected(L):
    st = None
    need = L.dust_layer_estimate_workspace(4, 16, 8, 0, 0.9)
    assert need >= 4 * 16 * 4 + 256
    assert status(L.dust_layer_estimate(GOOD, 0, 16, 8, GOOD, 1, 0.9, NZ.c(), GOOD, None, 0, GOOD, need - 1, st)) == 4
    need = L.dust_head_step_workspace(64, 32, 512, 128, 4, 1, 0, 1)
    assert need >= 64 * 512 * 4
    assert status(L.dust_head_step(GOOD, GOOD, 1, None, GOOD, 64, 32, 512, 128, 0, 4, NZ.c(), None, GOOD, None, GOOD,
                                   0, GOOD, need - 1, st)) == 4


def test_workspace_queries_are_consistent(L):
    # no scan needed -> status block only; scan needed -> room for r
    assert L.dust_layer_estimate_workspace(8, 100, 16, 1, 0.9) == 256
    assert L.dust_layer_estimate_workspace(8, 100, 16, 0, 0.0) == 256
    assert L.dust_layer_estimate_workspace(8, 100, 16, 0, 0.9) >= 256 + 8 * 100 * 4
    # cached Z needs no logits buffer
    assert L.dust_head_step_workspace(64, 32, 512, 128, 4, 1, 1, 0) < L.dust_head_step_workspace(64, 32, 512, 128, 4,
                                                                                                  1, 0, 0)


def test_fused_estimate_rejected_on_host(L):
    """dust_layer_estimate_weight_grad: d_in outside {64, ..., 512} step 64 is
    unsupported, bad sizes / pointers / workspaces are rejected before launch."""
    st = None
    f = L.dust_layer_estimate_weight_grad
    need = L.dust_layer_estimate_weight_grad_workspace(4, 96, 128, 40, 1, 0.0)
    assert need > 256
    assert L.dust_layer_estimate_weight_grad_workspace(4, 96, 1024, 40, 1, 0.0) == 256      # unsupported d_in
    for d_in in (1024, 100, 0, 32):
        assert status(f(GOOD, 1, 96, 40, None, 1, 0.0, NZ.c(), GOOD, d_in, GOOD, 0, None, GOOD, 1 << 30, st)) == 2
    assert status(f(GOOD, 1, 0, 40, None, 1, 0.0, NZ.c(), GOOD, 128, GOOD, 0, None, GOOD, 1 << 30, st)) == 1
    assert status(f(GOOD, 1, 96, 40, None, 1, 0.0, NZ.c(), GOOD + 8, 128, GOOD, 0, None, GOOD, 1 << 30, st)) == 3
    assert status(f(GOOD, 1, 96, 40, None, 1, 0.0, NZ.c(), GOOD, 128, None, 0, None, GOOD, 1 << 30, st)) == 1
    assert status(f(GOOD, 1, 96, 40, None, 1, 0.0, NZ.c(), GOOD, 128, GOOD, 0, None, GOOD, need - 1, st)) == 4
    need_scan = L.dust_layer_estimate_weight_grad_workspace(4, 96, 128, 40, 0, 0.9)
    assert need_scan >= need + 4 * 96 * 4
    # one call takes at most 2^20 draws (its bounded waits scale with the draw count)
    big = dust.Noise(0, 0, 0, (1 << 20) + 1, (1 << 20) + 1, 0.01).c()
    assert status(f(GOOD, 1, 1, 40, None, 1, 0.0, big, GOOD, 128, GOOD, 0, None, GOOD, 1 << 30, st)) == 2
    assert "accumulate" in L.dust_last_error().decode()


def test_binding_rejects_host_tensors():
    import torch
    with pytest.raises(ValueError):
        dust.reward_scan(torch.zeros(2, 8), torch.zeros(2, dtype=torch.int32), 0.5)
