"""Shared helpers for the GPU tests: input transfer, running the oracle, comparing."""
from __future__ import annotations

import numpy as np

from oracle import StreamOracle, bf16_bits_to_f64
from streaming_kv_cache_stream_b200.inputs import WORKLOADS, verify_inputs, window_inputs

MAX_ABS = 1e-2        # parity bar on attention outputs (bf16 in, fp32 accumulate)
REL_FRO = 5e-3


def to_dev(bits: np.ndarray):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev(t) -> np.ndarray:
    """Device output (fp32) to float64 on the host."""
    return t.detach().cpu().numpy().astype(np.float64)


def out_like(Q):
    import torch

    return torch.empty(Q.shape, dtype=torch.float32, device=Q.device)


def f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f64(bits)


def compare(got: np.ndarray, want: np.ndarray, what: str = "") -> dict:
    err = np.abs(got - want)
    mx = float(err.max()) if err.size else 0.0
    fro = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert mx <= MAX_ABS, f"{what}: max-abs {mx:.3e} > {MAX_ABS}"
    assert fro <= REL_FRO, f"{what}: rel-Frobenius {fro:.3e} > {REL_FRO}"
    return dict(max_abs=mx, rel_fro=fro)


def make_oracle(wl) -> StreamOracle:
    return StreamOracle(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d, wl.rope_base)


def make_stream(wl):
    from streaming_kv_cache_stream_b200.abi import Stream

    return Stream(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d, wl.rope_base)


def check_cache_bitexact(stream, orc: StreamOracle, wl) -> None:
    """Physical device rows vs the oracle's window, matched by (view, frame_id, token)."""
    ex = stream.debug_export()
    c = orc.cache_rows()
    n, T, V = wl.tok_per_frame, wl.frames, wl.views
    ring = V * T * n
    # oracle lookup: (view, frame_id, token) -> window row
    idx = {}
    for row, (v, f, t) in enumerate(zip(c["view"], c["frame_id"], c["token"])):
        idx[(int(v), int(f), int(t))] = row
    rows = ex["pos"].shape[0]
    assert rows == c["K"].shape[0], f"device holds {rows} rows, oracle {c['K'].shape[0]}"
    L = ring + wl.text_len
    want_rows = np.empty(rows, dtype=np.int64)
    for r in range(rows):
        if r < ring:
            v = r // (T * n)
            t = r % n
            want_rows[r] = idx[(v, int(ex["frame_id"][r]), t)]
        elif r < L:
            want_rows[r] = idx[(-1, -1, r - ring)]
        else:  # decode tail
            want_rows[r] = idx[(-2, -1, r - L)]
    # positions: bit-exact
    np.testing.assert_array_equal(ex["pos"], c["pos"][want_rows])
    # contents: the bf16 bit patterns themselves (the oracle holds exact upcasts of them)
    for name in ("K", "V"):
        want = np.transpose(c[name][want_rows], (1, 0, 2)).astype(np.float32).view(np.uint32) >> np.uint32(16)
        np.testing.assert_array_equal(ex[name], want.astype(np.uint16), err_msg=f"cache {name} bits")


__all__ = ["WORKLOADS", "window_inputs", "verify_inputs", "to_dev", "from_dev", "out_like", "f64", "compare", "make_oracle",
           "make_stream", "check_cache_bitexact", "MAX_ABS", "REL_FRO"]
