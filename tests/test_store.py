"""Saving and loading compressed layers (host side, no GPU): the planes come
back bit for bit, and every inconsistency or corruption is refused."""
import json
import os

import numpy as np
import pytest

from prng_seeded_decompress_b200 import inputs, store


@pytest.mark.parametrize("cp,rows,cols", [(inputs.FORMAT_4BIT, 7, 100),
                                          (inputs.FORMAT_3BIT, 5, 61)])
def test_roundtrip_is_bit_exact(tmp_path, oracle_mod, cp, rows, cols):
    L = inputs.make_layer(rows, cols, *cp, seed=3)
    prefix = str(tmp_path / "layer0")
    desc = store.save_layer(prefix, L["fmt"], L["rec"], L["eplane"])
    assert desc["format"] == L["fmt"]
    fmt, rec, ep = store.load_layer(prefix)
    assert fmt == L["fmt"]
    assert rec.dtype == np.uint32 and np.array_equal(rec, L["rec"])
    if cp[1] == 4:
        assert ep.dtype == np.uint8 and np.array_equal(ep, L["eplane"])
    else:
        assert ep is None
    # The loaded planes rebuild the same weights.
    assert np.array_equal(oracle_mod.decompress(fmt, rec, ep),
                          oracle_mod.decompress(L["fmt"], L["rec"], L["eplane"]))


def test_int32_records_are_accepted_as_their_bits(tmp_path):
    L = inputs.make_layer(3, 40, *inputs.FORMAT_4BIT, seed=4)
    store.save_layer(str(tmp_path / "a"), L["fmt"], L["rec"].view(np.int32))
    _, rec, _ = store.load_layer(str(tmp_path / "a"))
    assert np.array_equal(rec, L["rec"])


def test_corruption_and_mismatches_are_refused(tmp_path):
    L = inputs.make_layer(4, 48, *inputs.FORMAT_3BIT, seed=5)
    prefix = str(tmp_path / "b")
    store.save_layer(prefix, L["fmt"], L["rec"], L["eplane"])
    # One flipped byte in a plane.
    path = prefix + ".rec.bin"
    data = bytearray(open(path, "rb").read())
    data[5] ^= 1
    open(path, "wb").write(bytes(data))
    with pytest.raises(ValueError, match="SHA-256"):
        store.load_layer(prefix)
    # A truncated plane.
    open(path, "wb").write(bytes(data[:-4]))
    with pytest.raises(ValueError, match="bytes on disk"):
        store.load_layer(prefix)
    # A description whose format does not hold together.
    store.save_layer(prefix, L["fmt"], L["rec"], L["eplane"])
    desc = json.load(open(prefix + ".json"))
    desc["format"]["nb"] += 1
    json.dump(desc, open(prefix + ".json", "w"))
    with pytest.raises(ValueError, match="nb"):
        store.load_layer(prefix)
    # A plane file outside the folder.
    store.save_layer(prefix, L["fmt"], L["rec"], L["eplane"])
    desc = json.load(open(prefix + ".json"))
    desc["planes"]["rec"]["file"] = os.path.join("..", "x.bin")
    json.dump(desc, open(prefix + ".json", "w"))
    with pytest.raises(ValueError, match="next to the description"):
        store.load_layer(prefix)


def test_save_refuses_inconsistent_inputs(tmp_path):
    L4 = inputs.make_layer(2, 16, *inputs.FORMAT_4BIT, seed=6)
    L3 = inputs.make_layer(2, 24, *inputs.FORMAT_3BIT, seed=6)
    with pytest.raises(ValueError, match="no exponent plane"):
        store.save_layer(str(tmp_path / "c"), L4["fmt"], L4["rec"], np.zeros((2, 16), np.uint8))
    with pytest.raises(ValueError, match="needs its exponent plane"):
        store.save_layer(str(tmp_path / "c"), L3["fmt"], L3["rec"])
    with pytest.raises(ValueError, match="elements"):
        store.save_layer(str(tmp_path / "c"), L4["fmt"], L4["rec"][:1])
    with pytest.raises(ValueError, match="unsupported"):
        store.save_layer(str(tmp_path / "c"), dict(L4["fmt"], P=4), L4["rec"])
    with pytest.raises(ValueError, match="expected uint32"):
        store.save_layer(str(tmp_path / "c"), L4["fmt"], L4["rec"].astype(np.float32))
