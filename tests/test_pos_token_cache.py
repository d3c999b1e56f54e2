"""Host logic of the position-token cache, on the CPU (the token kernel is
replaced by a counting stand-in that returns a fresh object per call)."""
import gc
import weakref

import pytest
import torch

import windowed_attention_implicit_b200 as R

HEADS, RANK, HID, F = 2, 4, 6, 3


def _mlp():
    t = lambda *s: torch.randn(*s)
    return R.PositionMLP(t(F), t(HID, 4 * F), t(HID), t(HEADS * RANK, HID), t(HEADS * RANK),
                         t(HID, 4 * F), t(HID), t(HEADS * RANK, HID), t(HEADS * RANK),
                         HEADS, RANK)


@pytest.fixture
def calls(monkeypatch):
    log = []

    def fake(mlp, window, stream=None):
        log.append(window)
        return ("tokens", len(log))
    monkeypatch.setattr(R, "rib_pos_tokens", fake)
    return log


def test_one_computation_per_geometry(calls):
    cache, mlp = R.PosTokenCache(), _mlp()
    a = cache.get(mlp, 16)
    assert cache.get(mlp, 16) is a
    b = cache.get(mlp, 32)
    assert b is not a and calls == [16, 32] and len(cache) == 2
    # another record over the very same tensors is the same MLP
    same = R.PositionMLP(*mlp.tensors(), HEADS, RANK)
    assert cache.get(same, 16) is a and calls == [16, 32]


def test_in_place_updates_recompute_and_replace(calls):
    cache, mlp = R.PosTokenCache(), _mlp()
    a = cache.get(mlp, 16)
    with torch.no_grad():
        mlp.q_w1.add_(0.1)                     # an optimizer step on a weight
    b = cache.get(mlp, 16)
    assert b is not a and calls == [16, 16] and len(cache) == 1
    assert cache.get(mlp, 16) is b
    mlp.k_b2.mul_(2.0)                         # a bias counts too
    c = cache.get(mlp, 16)
    assert c is not b and len(calls) == 3 and len(cache) == 1
    mlp.freqs.fill_(1.0)                       # and the frequencies
    assert cache.get(mlp, 16) is not c and len(calls) == 4


def test_equal_values_in_other_tensors_are_another_entry(calls):
    cache, mlp = R.PosTokenCache(), _mlp()
    cache.get(mlp, 16)
    twin = R.PositionMLP(*(t.clone() for t in mlp.tensors()), HEADS, RANK)
    cache.get(twin, 16)
    assert len(calls) == 2 and len(cache) == 2


def test_entry_keeps_its_tensors_alive(calls):
    cache, mlp = R.PosTokenCache(), _mlp()
    cache.get(mlp, 16)
    ref = weakref.ref(mlp.q_w2)
    del mlp
    gc.collect()
    assert ref() is not None                   # its address cannot be reused
    cache.clear()
    gc.collect()
    assert ref() is None and len(cache) == 0


def test_inference_mode_tensors(calls):
    with torch.inference_mode():
        mlp = _mlp()
    cache = R.PosTokenCache()
    a = cache.get(mlp, 16)
    assert cache.get(mlp, 16) is a and calls == [16]
    assert mlp.versions() == (-1,) * 9
