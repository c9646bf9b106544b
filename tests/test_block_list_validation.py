"""The host-side skip-list check (calib_validate_block_list_host), on the CPU: lists built
by the oracle's skip-list and schedule builders pass; each kind of malformed list that the
attention kernels would trust is refused.  No device work."""
import numpy as np
import pytest

import oracle
from calibrated_block_sparse_calib_b200 import ops


def _good(seed=0, H=3, nq=9, nk=13, p=0.3):
    rng = np.random.default_rng(seed)
    m = (rng.random((H, nq, nk)) < p).astype(np.uint8)
    m[0, 0] = 0                                            # an empty row is valid
    rp, ci = oracle.mask_to_csr(m)
    work = oracle.build_schedule(rp, H, nq)
    return H, nq, nk, rp, ci, work


def test_lists_from_the_builders_pass():
    for seed in range(5):
        H, nq, nk, rp, ci, work = _good(seed)
        assert ops.validate_block_list_host(H, nq, nk, rp, ci, work)
        assert ops.validate_block_list_host(H, nq, nk, rp, ci)          # no work list
    # a list with no kept block at all, and the dense one
    H, nq, nk = 2, 4, 4
    assert ops.validate_block_list_host(H, nq, nk, np.zeros(H * nq + 1, np.int32), np.zeros(0, np.int16))
    rp, ci = oracle.mask_to_csr(np.ones((H, nq, nk), np.uint8))
    assert ops.validate_block_list_host(H, nq, nk, rp, ci, oracle.build_schedule(rp, H, nq))


def _mutations():
    H, nq, nk, rp, ci, work = _good(11)
    r = int(np.argmax(np.diff(rp)))                       # a row with kept blocks
    b, e = int(rp[r]), int(rp[r + 1])
    assert e - b >= 2
    cases = {}
    x = rp.copy(); x[0] = 1; cases["row_ptr[0] != 0"] = (x, ci, work)
    x = rp.copy(); x[r + 1] = x[r] - 1; cases["decreasing row pointers"] = (x, ci, work)
    x = rp.copy(); x[-1] = len(ci) + 1; cases["last row past col_idx"] = (x, ci, work)
    x = rp.copy(); x[1:] += 0; x[-1] = x[-2] + nk + 1; cases["a row longer than nk"] = (x, np.zeros(x[-1], np.int16), work)
    y = ci.copy(); y[b] = nk; cases["index == nk"] = (rp, y, work)
    y = ci.copy(); y[b] = -1; cases["negative index"] = (rp, y, work)
    y = ci.copy(); y[b + 1] = y[b]; cases["repeated index"] = (rp, y, work)
    y = ci.copy(); y[b], y[b + 1] = y[b + 1], y[b]; cases["descending indices"] = (rp, y, work)
    w = work.copy(); w[3] = (H << 16) | 0; cases["work head == H"] = (rp, ci, w)
    w = work.copy(); w[3] = (0 << 16) | nq; cases["work query block == nq"] = (rp, ci, w)
    w = work.copy(); w[3] = -1; cases["negative work item"] = (rp, ci, w)
    return H, nq, nk, cases


@pytest.mark.parametrize("name", list(_mutations()[3]))
def test_malformed_lists_are_refused(name):
    H, nq, nk, cases = _mutations()
    rp, ci, work = cases[name]
    assert not ops.validate_block_list_host(H, nq, nk, rp, ci, work), name


def test_shape_errors_are_refused():
    H, nq, nk, rp, ci, work = _good(2)
    assert not ops.validate_block_list_host(H, nq, nk, rp[:-1], ci, work)      # row_ptr too short
    assert not ops.validate_block_list_host(H, nq, 0, rp, ci, work)            # nk < 1
    assert not ops.validate_block_list_host(H, nq, 40000, rp, ci, work)        # nk beyond int16
