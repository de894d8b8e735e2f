"""GPU parity of the vision encoder's attention over each view's newest frame
(fs_frame_attend) against the fp64 oracle (frame_attention): max-abs 1e-2,
relative Frobenius 5e-3."""
from __future__ import annotations

import numpy as np
import pytest

from helpers import compare, f64, from_dev, make_stream, to_dev
from oracle import frame_attention
from streaming_kv_cache_stream_b200.inputs import WORKLOADS, Workload, f32_to_bf16_bits, frame_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from streaming_kv_cache_stream_b200 import abi

    abi.load()


def _run(wl, Qb, Kb, Vb):
    import torch

    s = make_stream(wl)
    Q, K, V = to_dev(Qb), to_dev(Kb), to_dev(Vb)
    out = torch.empty(Q.shape, dtype=torch.float32, device="cuda")
    s.frame_attend(Q, K, V, out)
    s.sync()
    got = from_dev(out)
    s.close()
    return got


@pytest.mark.parametrize("wid", [2, 3, 4])
def test_frame_attention_workload_shapes(wid):
    """The newest frames of the medium, driving and wide windows (64, 180 and 256
    tokens per frame), encoder heads 16 x 64."""
    wl = WORKLOADS[wid]
    b = frame_inputs(wid, 0, 1)
    got = _run(wl, b["Q"], b["K"], b["V"])
    compare(got, frame_attention(f64(b["Q"]), f64(b["K"]), f64(b["V"]), wl.views, wl.tok_per_frame),
            f"frame attention, workload {wid}")


@pytest.mark.parametrize("views,n,H,Hkv,d", [
    (1, 1, 4, 4, 64),       # one token
    (3, 128, 8, 8, 128),    # exactly one key tile
    (2, 129, 32, 8, 128),   # ragged second key tile, GQA
    (2, 300, 8, 1, 64),     # three key tiles, G = 8
    (7, 33, 2, 2, 128),     # seven views, short frames
])
def test_frame_attention_edge_shapes(views, n, H, Hkv, d):
    wl = Workload("frame-edge", views, 2, n, 0, H=H, Hkv=Hkv, d=d)
    rng = np.random.default_rng(views * 1000 + n)
    Qb = f32_to_bf16_bits(rng.standard_normal((views * n, H, d)).astype(np.float32))
    Kb = f32_to_bf16_bits((2 * rng.standard_normal((views * n, Hkv, d))).astype(np.float32))
    Vb = f32_to_bf16_bits(rng.standard_normal((views * n, Hkv, d)).astype(np.float32))
    got = _run(wl, Qb, Kb, Vb)
    compare(got, frame_attention(f64(Qb), f64(Kb), f64(Vb), views, n), f"frame {views}x{n} H{H}/{Hkv} d{d}")
