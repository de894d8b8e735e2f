"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Cache contents and positions must match bit for bit; attention outputs must be
within max-abs 1e-2 and relative Frobenius 5e-3 of the fp64 oracle (bf16 in,
fp32 accumulate, fp32 out). Inputs are the shared seeded bf16 draws.
"""
from __future__ import annotations

import numpy as np
import pytest

from helpers import (WORKLOADS, check_cache_bitexact, compare, f64, from_dev, make_oracle, make_stream, out_like, to_dev,
                     verify_inputs, window_inputs)
from streaming_kv_cache_stream_b200.inputs import Workload, f32_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from streaming_kv_cache_stream_b200 import abi

    abi.load()


def _run_steps(wid, layer=0, steps=None, rows_per_step=None, check_cache_every=1, full_last=False,
               check_out=True, check_cache_last=False):
    import torch

    wl = WORKLOADS[wid]
    steps = wl.steps if steps is None else steps
    s = make_stream(wl)
    orc = make_oracle(wl)
    stats = []
    for k in range(steps + 1):
        inp = window_inputs(wid, layer, k)
        Q, K, V = (to_dev(inp[x]) for x in ("Q", "K", "V"))
        out = out_like(Q)
        s.insert(K, V)
        s.attend(Q, out)
        torch.cuda.synchronize()
        nq = Q.shape[0]
        rows = None
        if rows_per_step is not None and not (full_last and k == steps):
            rng = np.random.default_rng([wid, layer, k])
            rows = np.unique(np.concatenate([[0, nq - 1], rng.choice(nq, size=min(rows_per_step, nq), replace=False)]))
        Kf, Vf = f64(inp["K"]), f64(inp["V"])
        if check_out:
            Qf = f64(inp["Q"])
            want = orc.prefill(Qf, Kf, Vf, rows=rows) if k == 0 else orc.step(Qf, Kf, Vf, rows=rows)
            got = from_dev(out)
            if rows is not None:
                got = got[rows]
            stats.append(compare(got, want, f"workload {wid} layer {layer} step {k}"))
        else:
            (orc.win.prefill if k == 0 else orc.win.step)(Kf, Vf)
            assert np.isfinite(from_dev(out)).all()
        if (check_cache_every and k % check_cache_every == 0) or (check_cache_last and k == steps):
            check_cache_bitexact(s, orc, wl)
    s.sync()
    s.close()
    return stats


def test_tiny_window_all_outputs():
    _run_steps(1, steps=3)


def test_medium_window_five_steps():
    _run_steps(2)


def test_driving_window_layers_sampled():
    # All 36 independent layers x 20 steps run on the GPU. Every layer's outputs are
    # compared on 12 sampled query rows (plus the first and last) of every step, the
    # rows drawn per (layer, step); the last step of layers 0 and 35 in full; every
    # layer's cache is checked bit-exact after its last step (layer 0's every 5 steps).
    wl = WORKLOADS[3]
    for layer in range(wl.layers):
        _run_steps(3, layer=layer, rows_per_step=12, check_cache_every=5 if layer == 0 else 0,
                   full_last=layer in (0, wl.layers - 1), check_out=True, check_cache_last=True)


def test_wide_window_outliers():
    # 14,848-key window with 1% outlier keys; every step sampled, the last step in full.
    _run_steps(4, rows_per_step=48, check_cache_every=5, full_last=True)


def test_verify_block_64_calls():
    import torch

    wl = WORKLOADS[5]
    s = make_stream(wl)
    orc = make_oracle(wl)
    for k in range(wl.steps + 1):  # the workload-2 cache after one full step
        inp = window_inputs(5, 0, k)
        Q, K, V = (to_dev(inp[x]) for x in ("Q", "K", "V"))
        out = out_like(Q)
        s.insert(K, V)
        s.attend(Q, out)
        Qf, Kf, Vf = f64(inp["Q"]), f64(inp["K"]), f64(inp["V"])
        orc.prefill(Qf, Kf, Vf) if k == 0 else orc.step(Qf, Kf, Vf)
    for call in range(wl.verify_calls):
        v = verify_inputs(5, call)
        Qx, Kx, Vx = (to_dev(v[x]) for x in ("Q", "K", "V"))
        out = out_like(Qx)
        s.attend_ext(Qx, Kx, Vx, out)
        torch.cuda.synchronize()
        want = orc.verify(f64(v["Q"]), f64(v["K"]), f64(v["V"]))
        compare(from_dev(out), want, f"verify call {call}")
    check_cache_bitexact(s, orc, wl)  # the drafted blocks left the window untouched
    s.sync()
    s.close()


EDGE_SHAPES = [
    # (views, frames, tok_per_frame, text_len, H, Hkv, d, steps)
    (1, 1, 16, 0, 4, 4, 128, 2),     # T = 1, one view, no text, G = 1
    (1, 4, 40, 0, 8, 1, 64, 5),      # one view, plain causal over frames, G = 8
    (3, 3, 1, 5, 8, 2, 128, 4),      # one token per frame
    (2, 5, 77, 3, 16, 4, 128, 6),    # ragged tiles everywhere, ring wraps past T
    (5, 2, 33, 130, 32, 8, 64, 3),   # text spans more than one key tile, d = 64
    (2, 2, 200, 1, 2, 2, 128, 3),    # G = 1, frames longer than a tile
]


@pytest.mark.parametrize("shape", EDGE_SHAPES, ids=[str(s) for s in EDGE_SHAPES])
def test_edge_shapes(shape):
    import torch

    V_, T, n, X, H, Hkv, d, steps = shape
    wl = Workload("edge", V_, T, n, X, H=H, Hkv=Hkv, d=d, steps=steps)
    s = make_stream(wl)
    orc = make_oracle(wl)
    rng = np.random.default_rng(hash(shape) & 0xFFFF)
    for k in range(steps + 1):
        N = wl.tokens(k)
        bits = {x: f32_to_bf16_bits(rng.standard_normal((N, H if x == "Q" else Hkv, d)).astype(np.float32))
                for x in ("Q", "K", "V")}
        Q, K, V = (to_dev(bits[x]) for x in ("Q", "K", "V"))
        out = out_like(Q)
        s.insert(K, V)
        s.attend(Q, out)
        torch.cuda.synchronize()
        Qf, Kf, Vf = f64(bits["Q"]), f64(bits["K"]), f64(bits["V"])
        want = orc.prefill(Qf, Kf, Vf) if k == 0 else orc.step(Qf, Kf, Vf)
        compare(from_dev(out), want, f"{shape} step {k}")
        check_cache_bitexact(s, orc, wl)
    # drafted blocks of 1 and of the maximum size
    for nx in (1, 256):
        bits = {x: f32_to_bf16_bits(rng.standard_normal((nx, H if x == "Q" else Hkv, d)).astype(np.float32))
                for x in ("Q", "K", "V")}
        Qx, Kx, Vx = (to_dev(bits[x]) for x in ("Q", "K", "V"))
        out = out_like(Qx)
        s.attend_ext(Qx, Kx, Vx, out)
        torch.cuda.synchronize()
        compare(from_dev(out), orc.verify(f64(bits["Q"]), f64(bits["K"]), f64(bits["V"])), f"{shape} verify {nx}")
    s.sync()
    s.close()


def test_verify_interleaved_with_steps():
    """Drafted blocks between window steps: a verify call leaves the window (and
    the next attend of the same queries) unchanged, and the next step rotates
    the whole window again. Medium window: prefill, step, verify, attend again,
    step, verify, attend."""
    import torch

    wl = WORKLOADS[2]
    s = make_stream(wl)
    orc = make_oracle(wl)
    for k in range(3):
        inp = window_inputs(2, 0, k)
        Q, K, V = (to_dev(inp[x]) for x in ("Q", "K", "V"))
        out = out_like(Q)
        s.insert(K, V)
        s.attend(Q, out)
        Qf, Kf, Vf = f64(inp["Q"]), f64(inp["K"]), f64(inp["V"])
        want = orc.prefill(Qf, Kf, Vf) if k == 0 else orc.step(Qf, Kf, Vf)
        torch.cuda.synchronize()
        compare(from_dev(out), want, f"step {k}")
        if k == 0:
            continue
        first = from_dev(out)
        for call in range(2):
            v = verify_inputs(5, 8 * k + call)
            Qx, Kx, Vx = (to_dev(v[x]) for x in ("Q", "K", "V"))
            ox = out_like(Qx)
            s.attend_ext(Qx, Kx, Vx, ox)
            torch.cuda.synchronize()
            compare(from_dev(ox), orc.verify(f64(v["Q"]), f64(v["K"]), f64(v["V"])), f"verify after step {k}")
        again = out_like(Q)
        s.attend(Q, again)
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(again), first), "a drafted block changed the next attend of the same queries"
    s.sync()
    check_cache_bitexact(s, orc, wl)
