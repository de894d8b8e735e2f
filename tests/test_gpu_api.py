"""C-ABI behaviour on the GPU: state machine, argument checks, the bounded-wait
error path, and the host-buffer step (fs_stream_step_host) against the device path."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

from helpers import WORKLOADS, compare, f64, from_dev, make_oracle, make_stream, to_dev, window_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from streaming_kv_cache_stream_b200 import abi

    abi.load()


def test_state_machine_and_errors():
    import torch

    from streaming_kv_cache_stream_b200 import abi

    wl = WORKLOADS[1]
    s = make_stream(wl)
    lib = abi.load()
    i = s.info()
    assert i.state == abi.FS_STATE_EXPECT_PREFILL and i.insert_tokens == wl.window_len and i.query_tokens == 0
    Q = torch.zeros(wl.window_len, wl.H, wl.d, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(Q.shape, dtype=torch.float32, device='cuda')
    with pytest.raises(abi.FsError) as e:
        s.attend(Q, out)
    assert e.value.code == abi.FS_ERR_STATE
    assert s.info().state == abi.FS_STATE_EXPECT_PREFILL
    # misaligned pointer is rejected and changes nothing
    K = torch.zeros(wl.window_len * wl.Hkv * wl.d + 8, dtype=torch.bfloat16, device="cuda")
    rc = lib.fs_stream_insert(s.handle, ctypes.c_void_p(K.data_ptr() + 2), ctypes.c_void_p(K.data_ptr() + 2))
    assert rc == abi.FS_ERR_ARG and s.info().state == abi.FS_STATE_EXPECT_PREFILL
    inp = window_inputs(1, 0, 0)
    s.insert(to_dev(inp["K"]), to_dev(inp["V"]))
    i = s.info()
    assert i.state == abi.FS_STATE_PREFILLED and i.query_tokens == wl.window_len and i.head == 0
    s.attend(to_dev(inp["Q"]), out)
    inp1 = window_inputs(1, 0, 1)
    s.insert(to_dev(inp1["K"]), to_dev(inp1["V"]))
    i = s.info()
    assert i.state == abi.FS_STATE_STREAMING and i.head == 1 % wl.frames and i.steps == 1
    assert i.insert_tokens == wl.step_tokens == i.query_tokens
    Qx = to_dev(inp1["Q"][:1])
    with pytest.raises(abi.FsError) as e:  # output aliasing the queries is rejected
        s.attend_ext(Qx, to_dev(inp1["K"][:1]), to_dev(inp1["V"][:1]), Qx.view(torch.float32)[:, :16])
    assert e.value.code == abi.FS_ERR_ARG
    assert s.info().steps == 1
    s.reset()
    assert s.info().state == abi.FS_STATE_EXPECT_PREFILL
    s.sync()
    s.close()


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch

    from streaming_kv_cache_stream_b200 import abi

    wl = WORKLOADS[1]
    s = make_stream(wl)
    lib = abi.load()
    rc = lib.fs_stream_debug_wait_probe(s.handle, 2000)  # 2 ms limit on a barrier nobody completes
    assert rc == abi.FS_ERR_DEVICE_TIMEOUT
    assert b"bounded" in lib.fs_stream_last_error(s.handle)
    # the flag was cleared and the context still works
    assert lib.fs_stream_sync(s.handle) == abi.FS_OK
    inp = window_inputs(1, 0, 0)
    out = torch.empty(wl.window_len, wl.H, wl.d, dtype=torch.float32, device="cuda")
    s.insert(to_dev(inp["K"]), to_dev(inp["V"]))
    s.attend(to_dev(inp["Q"]), out)
    s.sync()
    orc = make_oracle(wl)
    compare(from_dev(out), orc.prefill(f64(inp["Q"]), f64(inp["K"]), f64(inp["V"])), "after probe")
    s.close()


def test_host_buffer_step_matches_device_path():
    import torch

    wl = WORKLOADS[2]
    a = make_stream(wl)
    b = make_stream(wl)
    for k in range(3):
        inp = window_inputs(2, 0, k)
        out_d = torch.empty(inp["Q"].shape, dtype=torch.float32, device="cuda")
        a.insert(to_dev(inp["K"]), to_dev(inp["V"]))
        a.attend(to_dev(inp["Q"]), out_d)
        pin = {x: torch.from_numpy(inp[x].view(np.int16)).pin_memory() for x in ("Q", "K", "V")}
        out_h = torch.empty(inp["Q"].shape, dtype=torch.float32).pin_memory()
        b.step_host(pin["K"], pin["V"], pin["Q"], out_h)
        b.sync()
        a.sync()
        assert torch.equal(out_d.cpu(), out_h), f"step {k}"
    a.close()
    b.close()
