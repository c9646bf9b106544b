"""The mask dictionary's file format, round-tripped on the CPU with oracle-made slices
(no kernel involved): every array, flag and header field survives, and damaged files are
rejected."""
import struct

import numpy as np
import pytest
import torch

import oracle
from calibrated_block_sparse_calib_b200.dictionary import MaskDictionary, _Slice, MAGIC


def _dict(seed=0):
    rng = np.random.default_rng(seed)
    T, L, H, nq, nk = 3, 2, 3, 7, 11
    d = MaskDictionary(T, L, H, nq, nk, block=64, stride=4)
    ref = {}
    for t in range(T):
        for l in range(L):
            if (t, l) == (2, 1):
                continue                                  # a missing slice stays missing
            m = (rng.random((H, nq, nk)) < 0.1 + 0.3 * t).astype(np.uint8)
            ip, st, ln = oracle.csr_to_intervals(*oracle.mask_to_csr(m))
            rep = tuple(bool(x) for x in rng.random(H) < 0.5)
            d.slices[(t, l)] = _Slice(torch.from_numpy(ip), torch.from_numpy(st), torch.from_numpy(ln), rep)
            ref[(t, l)] = (m, ip, st, ln, rep)
    return d, ref


def test_round_trip_every_field():
    d, ref = _dict()
    buf = d.to_bytes()
    assert buf[:8] == MAGIC
    e = MaskDictionary.from_bytes(buf, device="cpu")
    assert (e.T, e.L, e.H, e.nq, e.nk, e.block, e.stride) == (3, 2, 3, 7, 11, 64, 4)
    assert set(e.slices) == set(ref)
    for key, (m, ip, st, ln, rep) in ref.items():
        s = e.slices[key]
        np.testing.assert_array_equal(s.iv_ptr.numpy(), ip)
        np.testing.assert_array_equal(s.starts.numpy(), st)
        np.testing.assert_array_equal(s.lens.numpy(), ln)
        assert s.repeat == rep
        # the runs still describe the original mask
        rp, ci = oracle.intervals_to_csr(s.iv_ptr.numpy(), s.starts.numpy(), s.lens.numpy())
        np.testing.assert_array_equal((rp, ci)[0], oracle.mask_to_csr(m)[0])
        np.testing.assert_array_equal(ci, oracle.mask_to_csr(m)[1])
    assert e.to_bytes() == buf


def test_damaged_files_are_rejected():
    d, _ = _dict(1)
    buf = d.to_bytes()
    with pytest.raises(ValueError):
        MaskDictionary.from_bytes(b"XXXXXXXX" + buf[8:], device="cpu")
    with pytest.raises(ValueError):
        MaskDictionary.from_bytes(buf + b"\0\0\0\0", device="cpu")
    with pytest.raises(Exception):
        MaskDictionary.from_bytes(buf[:-4], device="cpu")


def test_keys_outside_the_grid_are_rejected():
    d = MaskDictionary(2, 2, 1, 1, 1, 64)
    with pytest.raises(KeyError):
        d._check_key(2, 0)


def _one_slice_bytes(iv_ptr, starts, lens, H=1, nq=2, nk=8, block=64):
    d = MaskDictionary(1, 1, H, nq, nk, block)
    d.slices[(0, 0)] = _Slice(torch.tensor(iv_ptr, dtype=torch.int32), torch.tensor(starts, dtype=torch.int16),
                              torch.tensor(lens, dtype=torch.int16), (False,) * H)
    return d.to_bytes()


def test_run_structure_is_checked_before_upload():
    """A slice whose runs could not have come from a mask is refused on the host: the
    device expansion would otherwise write past the skip list it sizes from the runs."""
    good = _one_slice_bytes([0, 2, 3], [0, 4, 1], [2, 3, 7])
    e = MaskDictionary.from_bytes(good, device="cpu")
    assert e.slices[(0, 0)].lens.tolist() == [2, 3, 7]
    bad_cases = {
        "empty run": ([0, 2, 3], [0, 4, 1], [2, 0, 7]),
        "run past nk": ([0, 2, 3], [0, 4, 1], [2, 5, 7]),
        "negative start": ([0, 2, 3], [0, 4, -1], [2, 3, 7]),
        "overlapping runs": ([0, 2, 3], [0, 1, 1], [2, 3, 7]),
        "runs out of order": ([0, 2, 3], [4, 0, 1], [3, 2, 7]),
        "offsets not from 0": ([1, 2, 3], [0, 4, 1], [2, 3, 7]),
        "offsets decreasing": ([0, 4, 3], [0, 4, 1], [2, 3, 7]),
    }
    for name, (ip, st, ln) in bad_cases.items():
        with pytest.raises(ValueError):
            MaskDictionary.from_bytes(_one_slice_bytes(ip, st, ln), device="cpu")


def test_bad_headers_are_refused():
    buf = bytearray(_one_slice_bytes([0, 1, 1], [0], [1]))
    for field, value in ((5, 96), (4, 0), (7, -1)):     # block 96, nk 0, n_slices -1
        b = bytearray(buf)
        struct.pack_into("<i", b, 8 + 4 * field, value)
        with pytest.raises(ValueError):
            MaskDictionary.from_bytes(bytes(b), device="cpu")
    b = bytearray(buf)
    struct.pack_into("<i", b, 64 + 8, -5)                # a negative run count
    with pytest.raises(ValueError):
        MaskDictionary.from_bytes(bytes(b), device="cpu")
    for field, value in ((8, 3), (9, 0), (10, 7), (11, -1)):   # rho 3/2, rho_den 0, mode 7, n_inputs -1
        b = bytearray(buf)
        struct.pack_into("<i", b, 8 + 4 * field, value)
        if field == 8:
            struct.pack_into("<i", b, 8 + 4 * 9, 2)
        with pytest.raises(ValueError):
            MaskDictionary.from_bytes(bytes(b), device="cpu")
    b = bytearray(buf)
    struct.pack_into("<d", b, 64 + 12, 1.5)              # a slice tau above 1
    with pytest.raises(ValueError):
        MaskDictionary.from_bytes(bytes(b), device="cpu")


def test_calibration_record_round_trips():
    """The file says how it was calibrated: the vote threshold rho, the aggregation mode,
    the number of inputs, the repetition threshold gamma and every slice's tau."""
    d, ref = _dict(3)
    d.rho, d.mode, d.n_inputs, d.gamma = (2, 3), "energy_mean", 4, 0.9
    for n, key in enumerate(sorted(d.slices)):
        d.slices[key].tau = [0.99, 0.95, 0.9][n % 3]
    e = MaskDictionary.from_bytes(d.to_bytes(), device="cpu")
    assert (e.rho, e.mode, e.n_inputs, e.gamma) == ((2, 3), "energy_mean", 4, 0.9)
    for n, key in enumerate(sorted(ref)):
        assert e.tau(*key) == [0.99, 0.95, 0.9][n % 3]
    d.gamma = None
    d.mode = "given"
    e = MaskDictionary.from_bytes(d.to_bytes(), device="cpu")
    assert e.gamma is None and e.mode == "given"


def test_first_format_is_refused_with_a_reason():
    d, _ = _dict(4)
    buf = b"CBSDICT1" + d.to_bytes()[8:]
    with pytest.raises(ValueError, match="CBSDICT1.*no calibration parameters"):
        MaskDictionary.from_bytes(buf, device="cpu")


def test_truncated_files_name_what_is_missing():
    d, _ = _dict(5)
    buf = d.to_bytes()
    for cut in (12, 60, 64 + 10, 64 + 20 + 3, len(buf) // 2, len(buf) - 2):
        with pytest.raises(ValueError, match="truncated|trailing|offsets|run"):
            MaskDictionary.from_bytes(buf[:cut], device="cpu")
    for cut in (12, 60, 64 + 10, 64 + 20 + 3):
        with pytest.raises(ValueError, match="truncated"):
            MaskDictionary.from_bytes(buf[:cut], device="cpu")


def test_skip_lists_beyond_int32_offsets_are_refused():
    """70000 rows, each one run of 32767 blocks: under 1 MB on disk, but the expanded skip
    list would hold 2.3e9 entries, past the int32 row offsets the device kernels use."""
    H, nq, nk = 1, 70000, 32767
    iv_ptr = np.arange(nq + 1, dtype="<i4")
    runs = np.zeros(nq, "<i2").tobytes() + np.full(nq, nk, "<i2").tobytes()
    buf = (MAGIC + struct.pack("<12i", 1, 1, H, nq, nk, 128, 1, 1, 1, 2, 0, 1) + struct.pack("<d", float("nan")) +
           struct.pack("<3id", 0, 0, nq, 0.9) + b"\1\0\0\0" + iv_ptr.tobytes() + runs)
    assert len(buf) < 1 << 20
    with pytest.raises(ValueError, match="2\\^31"):
        MaskDictionary.from_bytes(buf, device="cpu")
