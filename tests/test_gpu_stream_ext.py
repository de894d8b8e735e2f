"""GPU parity of the parts of the path beyond a plain window step, through the C ABI:

* re-base steps: keys are rotated once at a step-invariant angle index and the
  whole window is re-rotated every R-th step (R set through FS_REBASE_STEPS);
* fs_stream_insert_batch: one insert launch for a stack of layers, equal bit
  for bit to one fs_stream_insert per layer;
* the persisted decode tail: drafted-block verify, append of the accepted
  tokens, further verifies, then a window step that empties the tail;
* the supported input range: values just inside the fp16 operand limits match
  the oracle, and a value outside them is reported as FS_ERR_RANGE.
Outputs are compared with the fp64 oracle at max-abs 1e-2 / relative Frobenius
5e-3; cache contents and positions bit for bit."""
from __future__ import annotations

import os

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


class _rebase:
    """FS_REBASE_STEPS for the handles created inside the block."""

    def __init__(self, r):
        self.r = r

    def __enter__(self):
        self.old = os.environ.get("FS_REBASE_STEPS")
        os.environ["FS_REBASE_STEPS"] = str(self.r)

    def __exit__(self, *exc):
        if self.old is None:
            os.environ.pop("FS_REBASE_STEPS", None)
        else:
            os.environ["FS_REBASE_STEPS"] = self.old


def _bits(rng, n, heads, d, scale=1.0):
    return f32_to_bf16_bits((rng.standard_normal((n, heads, d)) * scale).astype(np.float32))


@pytest.mark.parametrize("R,shape", [
    (1, (2, 3, 40, 9, 8, 2, 128)),    # every step re-rotates the whole window
    (3, (2, 3, 40, 9, 8, 2, 128)),    # re-bases at steps 3 and 6
    (2, (3, 4, 33, 130, 16, 4, 64)),  # d = 64, text longer than a tile, re-bases at 2, 4, 6, 8
])
def test_rebase_steps_match_oracle(R, shape):
    import torch

    V_, T, n, X, H, Hkv, d = shape
    wl = Workload("rebase", V_, T, n, X, H=H, Hkv=Hkv, d=d, steps=9)
    with _rebase(R):
        s = make_stream(wl)
    assert s.info().rebase_every == R
    orc = make_oracle(wl)
    rng = np.random.default_rng(100 + R)
    for k in range(wl.steps + 1):
        N = wl.tokens(k)
        b = {"Q": _bits(rng, N, H, d), "K": _bits(rng, N, Hkv, d), "V": _bits(rng, N, Hkv, d)}
        Q, K, V = (to_dev(b[x]) for x in ("Q", "K", "V"))
        out = out_like(Q)
        s.insert(K, V)
        s.attend(Q, out)
        torch.cuda.synchronize()
        want = (orc.prefill if k == 0 else orc.step)(f64(b["Q"]), f64(b["K"]), f64(b["V"]))
        compare(from_dev(out), want, f"R={R} step {k}")
        check_cache_bitexact(s, orc, wl)
        # a drafted block after each step sees the same angle offsets
        nx = 5
        bx = {"Q": _bits(rng, nx, H, d), "K": _bits(rng, nx, Hkv, d), "V": _bits(rng, nx, Hkv, d)}
        ox = out_like(to_dev(bx["Q"]))
        s.attend_ext(to_dev(bx["Q"]), to_dev(bx["K"]), to_dev(bx["V"]), ox)
        torch.cuda.synchronize()
        compare(from_dev(ox), orc.verify(f64(bx["Q"]), f64(bx["K"]), f64(bx["V"])), f"R={R} verify after {k}")
    s.sync()
    s.close()


def test_insert_batch_equals_per_layer_inserts():
    """Three layers through one batched launch per step vs three single inserts,
    across two re-bases (R = 2): outputs and caches identical bit for bit."""
    import torch

    from streaming_kv_cache_stream_b200.abi import insert_batch

    wl = WORKLOADS[2]
    layers = 3
    with _rebase(2):
        a = [make_stream(wl) for _ in range(layers)]
        b = [make_stream(wl) for _ in range(layers)]
    orcs = [make_oracle(wl) for _ in range(layers)]
    for k in range(5):
        inps = [window_inputs(2, l, k) for l in range(layers)]
        dev = [{x: to_dev(inp[x]) for x in ("Q", "K", "V")} for inp in inps]
        insert_batch(a, [dv["K"] for dv in dev], [dv["V"] for dv in dev])
        outs_a = []
        for l in range(layers):
            o = out_like(dev[l]["Q"])
            a[l].attend(dev[l]["Q"], o)
            outs_a.append(o)
            b[l].insert(dev[l]["K"], dev[l]["V"])
            ob = out_like(dev[l]["Q"])
            b[l].attend(dev[l]["Q"], ob)
            torch.cuda.synchronize()
            assert torch.equal(o, ob), f"layer {l} step {k}: batched insert differs from the single insert"
            f = {x: f64(inps[l][x]) for x in ("Q", "K", "V")}
            want = (orcs[l].prefill if k == 0 else orcs[l].step)(f["Q"], f["K"], f["V"])
            if l == 1:
                compare(from_dev(o), want, f"batched layer {l} step {k}")
            check_cache_bitexact(a[l], orcs[l], wl)
        ia, ib = a[0].info(), b[0].info()
        assert ia.head == ib.head and ia.steps == ib.steps
    for s in a + b:
        s.sync()
        s.close()


def test_insert_batch_rejects_mixed_handles():
    from streaming_kv_cache_stream_b200.abi import FS_ERR_ARG, FS_ERR_STATE, FsError, insert_batch

    wl = WORKLOADS[1]
    s1, s2 = make_stream(wl), make_stream(wl)
    other = make_stream(WORKLOADS[2])
    inp = window_inputs(1, 0, 0)
    K, V = to_dev(inp["K"]), to_dev(inp["V"])
    with pytest.raises(FsError) as e:
        insert_batch([s1, s1], [K, K], [V, V])
    assert e.value.code == FS_ERR_ARG
    with pytest.raises(FsError) as e:
        insert_batch([s1, other], [K, K], [V, V])
    assert e.value.code == FS_ERR_ARG
    s1.insert(K, V)  # s1 past its prefill, s2 not
    with pytest.raises(FsError) as e:
        insert_batch([s1, s2], [K, K], [V, V])
    assert e.value.code == FS_ERR_STATE
    assert s2.info().state == 0
    for s in (s1, s2, other):
        s.sync()
        s.close()


def test_decode_tail_verify_append_step():
    """Verify -> append the accepted prefix -> verify -> ... -> window step, on
    the verify workload's cache (medium window), against the oracle; the tail is
    in the cache bit for bit and gone after the window step."""
    import torch

    wl = WORKLOADS[5]
    s = make_stream(wl)
    orc = make_oracle(wl)
    for k in range(wl.steps + 1):
        inp = window_inputs(5, 0, k)
        Q, K, V = (to_dev(inp[x]) for x in ("Q", "K", "V"))
        s.insert(K, V)
        s.attend(Q, out_like(Q))
        f = {x: f64(inp[x]) for x in ("Q", "K", "V")}
        (orc.prefill if k == 0 else orc.step)(f["Q"], f["K"], f["V"])
    accepted = [5, 8, 3, 6, 1]
    call = 0
    for rnd in range(2):
        for n_acc in accepted:
            v = verify_inputs(5, call)
            call += 1
            Qx, Kx, Vx = (to_dev(v[x]) for x in ("Q", "K", "V"))
            out = out_like(Qx)
            s.attend_ext(Qx, Kx, Vx, out)
            torch.cuda.synchronize()
            fx = {x: f64(v[x]) for x in ("Q", "K", "V")}
            compare(from_dev(out), orc.verify(fx["Q"], fx["K"], fx["V"]), f"round {rnd} call {call}")
            # the target accepts a prefix of the block: its K/V join the tail
            s.append(Kx[:n_acc].contiguous(), Vx[:n_acc].contiguous())
            orc.append(fx["K"][:n_acc], fx["V"][:n_acc])
            assert s.info().tail_tokens == orc.win.tail_len
        check_cache_bitexact(s, orc, wl)
        # next window: new frames and text, empty tail
        inp = window_inputs(5, 0, wl.steps + 1 + rnd)
        Q, K, V = (to_dev(inp[x]) for x in ("Q", "K", "V"))
        out = out_like(Q)
        s.insert(K, V)
        s.attend(Q, out)
        torch.cuda.synchronize()
        f = {x: f64(inp[x]) for x in ("Q", "K", "V")}
        compare(from_dev(out), orc.step(f["Q"], f["K"], f["V"]), f"window step after round {rnd}")
        assert s.info().tail_tokens == 0
        check_cache_bitexact(s, orc, wl)
    s.sync()
    s.close()


def test_decode_tail_limit():
    from streaming_kv_cache_stream_b200.abi import FS_ERR_ARG, FS_MAX_TAIL_TOKENS, FsError

    wl = WORKLOADS[1]
    s = make_stream(wl)
    inp = window_inputs(1, 0, 0)
    s.insert(to_dev(inp["K"]), to_dev(inp["V"]))
    rng = np.random.default_rng(3)
    big = to_dev(_bits(rng, FS_MAX_TAIL_TOKENS, wl.Hkv, wl.d))
    s.append(big, big)
    with pytest.raises(FsError) as e:
        s.append(big[:1].contiguous(), big[:1].contiguous())
    assert e.value.code == FS_ERR_ARG and s.info().tail_tokens == FS_MAX_TAIL_TOKENS
    s.sync()
    s.close()


def test_inputs_at_the_edge_of_the_fp16_range():
    """|V| up to 6e4, one key row per kv head reaching 4.6e4 (its rotated
    elements stay below 65504), queries reaching 3e5 (rotated and scaled by
    log2(e)/sqrt(128): below 65504): inside the supported range, so the output
    matches the oracle (relative to the output's scale) and no range error is
    raised."""
    import torch

    V_, T, n, X, H, Hkv, d = 2, 2, 64, 16, 8, 2, 128
    wl = Workload("range", V_, T, n, X, H=H, Hkv=Hkv, d=d, steps=2)
    s = make_stream(wl)
    orc = make_oracle(wl)
    rng = np.random.default_rng(21)
    for k in range(wl.steps + 1):
        N = wl.tokens(k)
        Vv = rng.standard_normal((N, Hkv, d)).astype(np.float32)
        Vv *= np.float32(60000.0) / np.abs(Vv).max()
        Kk = rng.standard_normal((N, Hkv, d)).astype(np.float32)
        Kk[N // 2, :, :] *= np.float32(46000.0) / np.abs(Kk[N // 2]).max()  # outlier key, |k| <= 4.6e4
        Qq = rng.standard_normal((N, H, d)).astype(np.float32)
        Qq *= np.float32(3.0e5) / np.abs(Qq).max()
        b = {"Q": f32_to_bf16_bits(Qq), "K": f32_to_bf16_bits(Kk), "V": f32_to_bf16_bits(Vv)}
        Q, K, V = (to_dev(b[x]) for x in ("Q", "K", "V"))
        out = out_like(Q)
        s.insert(K, V)
        s.attend(Q, out)
        s.sync()  # raises FS_ERR_RANGE if any element was flagged
        want = (orc.prefill if k == 0 else orc.step)(f64(b["Q"]), f64(b["K"]), f64(b["V"]))
        got = from_dev(out)
        assert np.isfinite(got).all()
        scale = float(np.abs(f64(b["V"])).max())
        err = float(np.abs(got - want).max())
        fro = float(np.linalg.norm(got - want) / np.linalg.norm(want))
        # P is fp16 (2^-11 relative) and V ~6e4: the bar scales with max|V|.
        assert err <= 1e-3 * scale and fro <= 5e-3, (k, err, scale, fro)
    s.close()


def test_out_of_range_input_is_reported():
    import torch

    from streaming_kv_cache_stream_b200.abi import FS_ERR_RANGE, FsError

    wl = WORKLOADS[1]
    s = make_stream(wl)
    inp = window_inputs(1, 0, 0)
    Vbits = inp["V"].copy()
    Vbits[3, 0, 5] = f32_to_bf16_bits(np.array([70000.0], dtype=np.float32))[0]  # above 65504
    s.insert(to_dev(inp["K"]), to_dev(Vbits))
    s.attend(to_dev(inp["Q"]), out_like(to_dev(inp["Q"])))
    with pytest.raises(FsError) as e:
        s.sync()
    assert e.value.code == FS_ERR_RANGE
    s.sync()  # the flag was cleared; the handle keeps working
    Qbits = inp["Q"].copy()
    Qbits[0, 0, 0] = f32_to_bf16_bits(np.array([1e6], dtype=np.float32))[0]  # scaled query above 65504
    s.reset()
    s.insert(to_dev(inp["K"]), to_dev(inp["V"]))
    s.attend(to_dev(Qbits), out_like(to_dev(Qbits)))
    with pytest.raises(FsError) as e:
        s.sync()
    assert e.value.code == FS_ERR_RANGE
    s.insert(to_dev(window_inputs(1, 0, 1)["K"]), to_dev(window_inputs(1, 0, 1)["V"]))
    s.sync()
    s.close()


@pytest.mark.parametrize("shape,nxs", [
    ((4, 4, 64, 32, 32, 8, 128), (1, 8, 31, 32, 33)),   # G = 4: one query tile up to 32 tokens, 33 takes the long path
    ((2, 3, 50, 7, 16, 2, 64), (1, 16, 17)),            # G = 8, d = 64
    ((1, 2, 100, 0, 4, 4, 128), (5, 128, 129)),         # G = 1, no text
])
def test_verify_block_sizes_against_oracle(shape, nxs):
    """Drafted blocks on both sides of the one-tile limit (n_x * G <= 128 runs
    the single-launch verify kernel), after a window step and with a decode
    tail, against the oracle."""
    import torch

    V_, T, n, X, H, Hkv, d = shape
    wl = Workload("verify-sizes", V_, T, n, X, H=H, Hkv=Hkv, d=d, steps=1)
    s = make_stream(wl)
    orc = make_oracle(wl)
    rng = np.random.default_rng(sum(shape))
    for k in range(2):
        N = wl.tokens(k)
        b = {"Q": _bits(rng, N, H, d), "K": _bits(rng, N, Hkv, d), "V": _bits(rng, N, Hkv, d)}
        s.insert(to_dev(b["K"]), to_dev(b["V"]))
        s.attend(to_dev(b["Q"]), out_like(to_dev(b["Q"])))
        (orc.prefill if k == 0 else orc.step)(f64(b["Q"]), f64(b["K"]), f64(b["V"]))
    for with_tail in (False, True):
        if with_tail:
            acc = {"K": _bits(rng, 11, Hkv, d), "V": _bits(rng, 11, Hkv, d)}
            s.append(to_dev(acc["K"]), to_dev(acc["V"]))
            orc.append(f64(acc["K"]), f64(acc["V"]))
        for nx in nxs:
            bx = {"Q": _bits(rng, nx, H, d), "K": _bits(rng, nx, Hkv, d), "V": _bits(rng, nx, Hkv, d)}
            Qx = to_dev(bx["Q"])
            ox = out_like(Qx)
            s.attend_ext(Qx, to_dev(bx["K"]), to_dev(bx["V"]), ox)
            torch.cuda.synchronize()
            compare(from_dev(ox), orc.verify(f64(bx["Q"]), f64(bx["K"]), f64(bx["V"])),
                    f"{shape} n_x={nx} tail={with_tail}")
    s.sync()
    check_cache_bitexact(s, orc, wl)
    s.close()


def test_verify_calls_replayed_from_a_cuda_graph():
    """Verify calls captured in a CUDA graph and replayed give the eager
    results bit for bit (no launch parameter depends on host state that the
    replay would freeze; the merge counters reset themselves)."""
    import torch

    wl = WORKLOADS[5]
    s = make_stream(wl)
    for k in range(wl.steps + 1):
        inp = window_inputs(5, 0, k)
        Q, K, V = (to_dev(inp[x]) for x in ("Q", "K", "V"))
        s.insert(K, V)
        s.attend(Q, out_like(Q))
    blocks = [{x: to_dev(verify_inputs(5, c)[x]) for x in ("Q", "K", "V")} for c in range(3)]
    eager = []
    for b in blocks:
        o = out_like(b["Q"])
        s.attend_ext(b["Q"], b["K"], b["V"], o)
        eager.append(o)
    torch.cuda.synchronize()
    outs = [out_like(b["Q"]) for b in blocks]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for b, o in zip(blocks, outs):
            s.attend_ext(b["Q"], b["K"], b["V"], o)
    for _ in range(3):
        for o in outs:
            o.zero_()
        g.replay()
        torch.cuda.synchronize()
        for o, e in zip(outs, eager):
            assert torch.equal(o, e)
    del g
    s.sync()
    s.close()
