"""Frozen lists on disk (bsa_lists_save / bsa_lists_read_header / bsa_lists_load): host
calls only, no GPU.  The lists are the method's only state between the calibration and
the later steps ("LoSA", Abstract: the selected block indices are frozen and reused), so a
saved file must give back exactly the lists that went in, and a damaged one must be
refused rather than read."""
import numpy as np
import pytest
import torch

from block_sparse_attention_25_b200 import synth

WL = synth.Workload("lists-6x10x11-h3", 2, 3, 128, 6, 10, 11, 8, 12, 12, 64, 64)


@pytest.fixture(scope="module")
def B():
    from block_sparse_attention_25_b200 import build
    build.build()
    import block_sparse_attention_25_b200 as b
    return b


def _lists(B, keep=0.4, seed=5):
    s = B.Shape.of(WL)
    rp, ci = synth.draw_keep_csr(s.rows, s.n_kb, keep, seed=seed, empty_rows=(0, 7))
    return s, rp, ci


def test_round_trip_is_exact(B, tmp_path):
    s, rp, ci = _lists(B)
    path = tmp_path / "lists.bin"
    B.save_lists(path, rp, ci, s, 0.99)
    rp2, ci2, tau = B.load_lists(path, s, device="cpu")
    assert torch.equal(rp2, rp) and torch.equal(ci2[:int(rp[-1])], ci)
    assert np.float32(tau) == np.float32(0.99)
    # a capacity-sized col_idx (as the selection returns it) saves the same file
    big = torch.full((s.rows * s.n_kb,), -1, dtype=torch.int32)
    big[:ci.numel()] = ci
    p2 = tmp_path / "lists2.bin"
    B.save_lists(p2, rp, big, s, 0.99)
    assert p2.read_bytes() == path.read_bytes()


def test_empty_lists_round_trip(B, tmp_path):
    s = B.Shape.of(WL)
    rp = torch.zeros(s.rows + 1, dtype=torch.int32)
    path = tmp_path / "empty.bin"
    B.save_lists(path, rp, torch.zeros(0, dtype=torch.int32), s, 0.5)
    rp2, ci2, _ = B.load_lists(path, s, device="cpu")
    assert torch.equal(rp2, rp) and ci2.numel() == 1


def test_damaged_files_are_refused(B, tmp_path):
    s, rp, ci = _lists(B)
    path = tmp_path / "lists.bin"
    B.save_lists(path, rp, ci, s, 0.99)
    good = path.read_bytes()

    def refused(data, status=7):
        bad = tmp_path / "bad.bin"
        bad.write_bytes(data)
        with pytest.raises(B.BsaError) as e:
            B.load_lists(bad, s, device="cpu")
        assert e.value.status == status

    refused(good[:-1])                                   # truncated hash
    refused(good[:200])                                  # truncated payload
    refused(good + b"\0")                                # trailing bytes
    refused(b"X" + good[1:])                             # magic
    flip = bytearray(good)
    flip[100] ^= 1                                       # one bit of row_ptr: hash mismatch
    refused(bytes(flip))
    with pytest.raises(B.BsaError) as e:                 # missing file
        B.load_lists(tmp_path / "nope.bin", s, device="cpu")
    assert e.value.status == 7
    other = B.Shape.of(WL.scaled(heads=2))               # lists of another shape
    with pytest.raises(B.BsaError) as e:
        B.load_lists(path, other, device="cpu")
    assert e.value.status in (1, 7)


def test_a_header_for_another_shape_sizes_no_buffer(B, tmp_path, monkeypatch):
    """A file whose (intact) header describes a much larger problem is refused by the shape
    comparison before the binding sizes any buffer from the header's entry count."""
    import ctypes
    big = B.Shape.of(synth.WORKLOADS["wan14b_720p"])
    rp = torch.arange(big.rows + 1, dtype=torch.int32) * big.n_kb   # every block kept
    path = tmp_path / "big.bin"
    # a header only: the payload is never reached
    B.save_lists(path, torch.zeros(big.rows + 1, dtype=torch.int32),
                 torch.zeros(0, dtype=torch.int32), big, 0.99)
    data = bytearray(path.read_bytes()[:80])
    data[72:80] = (int(rp[-1])).to_bytes(8, "little")                # 83 M entries claimed
    path.write_bytes(bytes(data) + b"\0" * 16)
    stored, tau, nnz = B.bsattn._Shape(), ctypes.c_float(), ctypes.c_int64()
    assert B.lib().bsa_lists_read_header(str(path).encode(), ctypes.byref(stored),
                                         ctypes.byref(tau), ctypes.byref(nnz)) == 0
    assert nnz.value == big.rows * big.n_kb
    sizes = []
    real_zeros = torch.zeros

    def counting_zeros(*a, **kw):
        sizes.append(a)
        return real_zeros(*a, **kw)

    monkeypatch.setattr(torch, "zeros", counting_zeros)
    s = B.Shape.of(WL)
    with pytest.raises(B.BsaError) as e:
        B.load_lists(path, s, device="cpu")
    assert e.value.status == 1 and sizes == []


def test_malformed_lists_are_not_saved(B, tmp_path):
    s, rp, ci = _lists(B)
    bad = ci.clone()
    r = int(torch.nonzero(rp[1:] - rp[:-1] >= 2)[0])    # a row with two entries
    b = int(rp[r])
    bad[b], bad[b + 1] = bad[b + 1].item(), bad[b].item()   # not ascending
    with pytest.raises(B.BsaError) as e:
        B.save_lists(tmp_path / "x.bin", rp, bad, s, 0.99)
    assert e.value.status == 1
    out = ci.clone()
    out[0] = s.n_kb                                      # out of range
    with pytest.raises(B.BsaError):
        B.save_lists(tmp_path / "x.bin", rp, out, s, 0.99)
    assert not (tmp_path / "x.bin").exists() and not (tmp_path / "x.bin.tmp").exists()


def test_fuzzed_files_are_refused_or_read_back_exactly(B, tmp_path):
    """400 seeded damages of a good file (bit flips anywhere, truncations, extensions, bytes
    overwritten in the header): the reader returns a status and never other lists."""
    s, rp, ci = _lists(B)
    path = tmp_path / "lists.bin"
    B.save_lists(path, rp, ci, s, 0.99)
    good = path.read_bytes()
    rng = np.random.default_rng(2024)
    bad = tmp_path / "fuzz.bin"
    for trial in range(400):
        data = bytearray(good)
        kind = trial % 4
        if kind == 0:
            for _ in range(int(rng.integers(1, 4))):
                i = int(rng.integers(0, len(data)))
                data[i] ^= 1 << int(rng.integers(0, 8))
        elif kind == 1:
            data = data[:int(rng.integers(0, len(data)))]
        elif kind == 2:
            data += bytes(rng.integers(0, 256, int(rng.integers(1, 64)), dtype=np.uint8))
        else:
            i = int(rng.integers(0, 80))
            data[i:i + 8] = bytes(rng.integers(0, 256, 8, dtype=np.uint8))
        bad.write_bytes(bytes(data))
        if bytes(data) == good:
            continue
        try:
            rp2, ci2, _ = B.load_lists(bad, s, device="cpu")
        except B.BsaError as e:
            assert e.status in (1, 3, 7), (trial, e.status)
            continue
        # only a change the hash does not cover could load; none exists, so: identical lists
        assert torch.equal(rp2, rp) and torch.equal(ci2[:int(rp[-1])], ci), trial
