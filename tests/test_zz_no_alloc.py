"""fs_stream_attend_ext_static (split-KV partials in the library's fixed device
array, no allocation) against fs_stream_attend_ext on the same inputs.

Collected last (file name) so that it runs both after every other GPU test and,
when selected alone, in a fresh process where its first call does the
per-device set-up of the array's address."""
from __future__ import annotations

import numpy as np
import pytest

from helpers import WORKLOADS, compare, from_dev, make_stream, out_like, to_dev, verify_inputs, window_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from streaming_kv_cache_stream_b200 import abi

    abi.load()


def _filled_verify_stream():
    """A stream holding the verify workload's cache (prefill + one window step)."""
    wl = WORKLOADS[5]
    s = make_stream(wl)
    for k in range(wl.steps + 1):
        inp = window_inputs(5, 0, k)
        Q, K, V = (to_dev(inp[x]) for x in ("Q", "K", "V"))
        s.insert(K, V)
        s.attend(Q, out_like(Q))
    return s


def _block(bits, n):
    return to_dev(np.ascontiguousarray(bits[:n]))


@pytest.mark.parametrize("n_x", [8, 96])
def test_static_scratch_matches_attend_ext_two_calls(n_x):
    """Two calls in a row of the static variant, each equal (within the parity
    tolerance) to fs_stream_attend_ext on the same block. n_x = 8 is the verify
    workload's block (same key splits on both paths); n_x = 96 needs 3 query
    tiles, where the static array caps the split count below the handle path's."""
    import torch

    s = _filled_verify_stream()
    blocks = []
    for call in range(2):
        if n_x == 8:
            v = verify_inputs(5, call)
        else:  # seeded window-step tensors, first n_x tokens, as a drafted block
            v = window_inputs(5, 0, 2 + call)
        blocks.append(tuple(_block(v[x], n_x) for x in ("Q", "K", "V")))
    ref = []
    for Qx, Kx, Vx in blocks:
        out = out_like(Qx)
        s.attend_ext(Qx, Kx, Vx, out)
        ref.append(out)
    got = []
    for Qx, Kx, Vx in blocks:  # back to back: the second call reuses the array the first one filled
        out = out_like(Qx)
        s.attend_ext_static(Qx, Kx, Vx, out)
        got.append(out)
    torch.cuda.synchronize()
    s.sync()
    for call in range(2):
        compare(from_dev(got[call]), from_dev(ref[call]), f"static vs attend_ext, n_x={n_x}, call {call}")


def test_static_scratch_rejects_calls_over_its_limit():
    """H/Hkv = 8, Hkv = 8: n_x = 256 needs 16 query tiles x 8 kv heads = 128
    partial tiles per split, over the array's 64; n_x = 64 (4 tiles) fits."""
    import torch

    from streaming_kv_cache_stream_b200.abi import FS_ERR_ARG, FsError, Stream

    s = Stream(1, 1, 16, 0, 64, 8, 64)
    rng = np.random.default_rng(7)

    def bf16(shape):
        return torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16).cuda()

    s.insert(bf16((16, 8, 64)), bf16((16, 8, 64)))
    s.attend(bf16((16, 64, 64)), torch.empty((16, 64, 64), dtype=torch.float32, device="cuda"))
    Qx, Kx, Vx = bf16((256, 64, 64)), bf16((256, 8, 64)), bf16((256, 8, 64))
    out = torch.empty((256, 64, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(FsError) as ei:
        s.attend_ext_static(Qx, Kx, Vx, out)
    assert ei.value.code == FS_ERR_ARG and "static split scratch" in str(ei.value)
    ref, got = out_like(Qx[:64]), out_like(Qx[:64])
    s.attend_ext(Qx[:64].contiguous(), Kx[:64].contiguous(), Vx[:64].contiguous(), ref)
    s.attend_ext_static(Qx[:64].contiguous(), Kx[:64].contiguous(), Vx[:64].contiguous(), got)
    torch.cuda.synchronize()
    s.sync()
    compare(from_dev(got), from_dev(ref), "static vs attend_ext, G=8, n_x=64")
