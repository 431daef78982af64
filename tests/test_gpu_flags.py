"""Device-side ordering between ranks: tide_flag_signal and tide_flag_wait, bounded waits.

Every wait here finds its flags already set by work ordered before it (earlier on the same
stream, or in another process that finished and met this one at a host barrier), or runs out
its time limit on a flag nothing sets; no two launches that wait on one another share the GPU.
A wait that runs out reports the late flag in its status word and the context stays usable.
"""
import json
import time

import pytest
import torch

from fsdp2_layout_aware_b200 import tide as T

from _dist_helpers import run_procs

pytestmark = pytest.mark.gpu


def _status():
    return torch.full((1,), -7, dtype=torch.int32, device="cuda")


def test_signal_then_wait_reports_the_first_late_flag():
    flags = torch.zeros(5, dtype=torch.int32, device="cuda")
    ptrs = [flags.data_ptr() + 4 * k for k in range(5)]
    for k, p in enumerate(ptrs):
        assert T.tide_flag_signal(p, 2 if k == 2 else 3) == T.TIDE_OK
    st = _status()
    assert T.tide_flag_wait(ptrs, 2, 10**9, st.data_ptr()) == T.TIDE_OK       # every flag >= 2
    torch.cuda.synchronize()
    assert st.item() == 0
    t0 = time.monotonic()
    assert T.tide_flag_wait(ptrs, 3, 20 * 10**6, st.data_ptr()) == T.TIDE_OK  # flag 2 stays at 2
    torch.cuda.synchronize()
    assert st.item() == 3 and time.monotonic() - t0 < 2.0
    assert flags.tolist() == [3, 3, 2, 3, 3]
    # the context is usable after a wait that ran out
    assert T.tide_flag_wait(ptrs[:2], 3, 10**9, st.data_ptr()) == T.TIDE_OK
    torch.cuda.synchronize()
    assert st.item() == 0


def test_epochs_compare_modulo_2_to_the_32():
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = _status()
    T.tide_flag_signal(flag.data_ptr(), 2)
    assert T.tide_flag_wait([flag.data_ptr()], 0xFFFFFFFE, 10**9, st.data_ptr()) == T.TIDE_OK
    torch.cuda.synchronize()
    assert st.item() == 0                        # 2 is four epochs after 2^32 - 2
    T.tide_flag_signal(flag.data_ptr(), 0xFFFFFFFF)
    assert T.tide_flag_wait([flag.data_ptr()], 1, 20 * 10**6, st.data_ptr()) == T.TIDE_OK
    torch.cuda.synchronize()
    assert st.item() == 1                        # 2^32 - 1 is two epochs before 1
    assert flag.item() == -1


def test_many_flags_one_late():
    n = T.TIDE_MAX_WORLD
    flags = torch.full((n,), 7, dtype=torch.int32, device="cuda")
    flags[200] = 6
    ptrs = [flags.data_ptr() + 4 * k for k in range(n)]
    st = _status()
    torch.cuda.synchronize()
    assert T.tide_flag_wait(ptrs, 7, 20 * 10**6, st.data_ptr()) == T.TIDE_OK
    torch.cuda.synchronize()
    assert st.item() == 201


def test_flags_across_processes_through_ipc(tmp_path):
    from _flag_workers import flag_worker
    run_procs(flag_worker, 2, lambda port: (port, str(tmp_path)))
    r0 = json.loads((tmp_path / "flags_0.json").read_text())
    r1 = json.loads((tmp_path / "flags_1.json").read_text())
    assert r0["signal"] == r1["wait_set"] == r1["wait_unset"] == r1["signal_peer"] == T.TIDE_OK
    assert r1["status_set"] == 0          # process 0's flag, set before the wait, seen through the mapping
    assert r1["status_unset"] == 2        # its flag 1 was not set yet: the wait ran out on index 1
    assert r0["wait_own"] == T.TIDE_OK and r0["status_own"] == 0
    assert r0["flags"] == [5, 9]          # process 1 set process 0's flag 1 through the mapping
