"""Checkpoint / resume of a layer-by-layer run (host logic, no GPU): each
finished linear's stored result goes to its own file, written whole or not
at all, and a restarted run quantizes only the linears without a file."""
import os

import pytest
import torch

import post_weight_quantization_25_b200 as G

NAMES = [f"b{b}.{l}" for b in range(2) for l in ("q", "k", "v", "o", "gate", "up", "down")]


def fake_quantize(calls, fail_on=None):
    def q(name):
        if name == fail_on:
            raise RuntimeError(f"stopped at {name}")
        calls.append(name)
        seed = NAMES.index(name)
        g = torch.Generator().manual_seed(seed)
        out = {"packed": torch.randint(-2 ** 31, 2 ** 31 - 1, (8, 4), generator=g,
                                       dtype=torch.int64).to(torch.int32),
               "scales": torch.rand(8, 1, generator=g), "zeros": torch.zeros(8, 1, dtype=torch.uint8),
               "g_idx": None, "perm": None}
        return out, {"name": name, "rows": 8, "n": 32, "bits": 4}
    return q


def test_resume_skips_finished_linears(tmp_path):
    d = str(tmp_path)
    calls = []
    with pytest.raises(RuntimeError):
        G.quantize_linears(NAMES, fake_quantize(calls, fail_on=NAMES[5]), d)
    assert calls == NAMES[:5]
    assert sorted(os.listdir(d)) == sorted(f"{n}.pt" for n in NAMES[:5])
    calls2 = []
    done = G.quantize_linears(NAMES, fake_quantize(calls2), d)
    assert calls2 == NAMES[5:] and done == NAMES[5:]
    # every stored result is the one its linear produced
    for name in NAMES:
        blob = G.load_quantized(os.path.join(d, f"{name}.pt"))
        ref, meta = fake_quantize([])(name)
        assert blob["meta"] == meta
        assert torch.equal(blob["packed"], ref["packed"])
        assert torch.equal(blob["scales"], ref["scales"])
        assert "g_idx" not in blob
    # nothing left to do
    calls3 = []
    assert G.quantize_linears(NAMES, fake_quantize(calls3), d) == [] and calls3 == []
    # without resume everything runs again
    calls4 = []
    assert G.quantize_linears(NAMES[:2], fake_quantize(calls4), d, resume=False) == NAMES[:2]


def test_interrupted_write_leaves_no_result(tmp_path, monkeypatch):
    """A run stopped while a file is being written leaves only the temporary
    file; the resumed run quantizes that linear again."""
    d = str(tmp_path)
    real_save = torch.save

    def broken_save(obj, path):
        with open(path, "wb") as f:
            f.write(b"partial")
        raise OSError("disk full")

    monkeypatch.setattr(torch, "save", broken_save)
    with pytest.raises(OSError):
        G.quantize_linears(NAMES[:1], fake_quantize([]), d)
    assert not os.path.exists(os.path.join(d, f"{NAMES[0]}.pt"))
    monkeypatch.setattr(torch, "save", real_save)
    calls = []
    assert G.quantize_linears(NAMES[:1], fake_quantize(calls), d) == NAMES[:1]
    assert calls == NAMES[:1]
