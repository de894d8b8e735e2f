"""Seeded synthetic inputs for the streaming KV-cache attention path.

This module only draws random numbers and rounds them to bf16. It holds none
of the method's arithmetic (no positions, no RoPE, no masking, no attention),
so both the CUDA path and the CPU oracle may take their inputs from it.

Every tensor is drawn from numpy's PCG64 seeded with
``SeedSequence([workload, layer, step, tensor, call])`` as float32 standard
normals, multiplied by the workload's scale, then rounded to bf16
(round-to-nearest-even). Tensor ids: Q = 0, K = 1, V = 2, outlier-row choice = 3;
the encoder attention's Q, K, V = 10, 11, 12; the hidden states and the K/V
projection weight = 20, 21.
Step 0 is the prefill window (the stream's first call); steps 1.. are window
steps; ``call`` numbers the verify calls.

The workload shapes stand in for the pages' 4-camera x 4-frame driving windows
(the PhysicalAI-AV clips the pages measure on are not used): see ``WORKLOADS``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

Q_ID, K_ID, V_ID, OUTLIER_ID = 0, 1, 2, 3
FRAME_Q_ID, FRAME_K_ID, FRAME_V_ID = 10, 11, 12  # encoder attention over the newest frames
X_ID, W_ID = 20, 21  # hidden states and the stacked K/V projection weight


@dataclass(frozen=True)
class Workload:
    """Shape of one synthetic streaming workload (sizes only)."""

    name: str
    views: int
    frames: int
    tok_per_frame: int
    text_len: int
    H: int
    Hkv: int
    d: int
    layers: int = 1
    steps: int = 1
    k_scale: float = 1.0
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    verify_calls: int = 0
    verify_tokens: int = 0
    cache_from: int | None = None  # workload id whose inputs fill the cache
    rope_base: float = 10000.0
    extra: dict = field(default_factory=dict)

    @property
    def window_len(self) -> int:
        return self.views * self.frames * self.tok_per_frame + self.text_len

    @property
    def step_tokens(self) -> int:
        return self.views * self.tok_per_frame + self.text_len

    def tokens(self, step: int) -> int:
        """Tokens inserted (and queries attended) at ``step``; step 0 is the prefill."""
        return self.window_len if step == 0 else self.step_tokens


WORKLOADS: dict[int, Workload] = {
    1: Workload("tiny", 2, 2, 16, 8, H=4, Hkv=2, d=64, layers=1, steps=1),
    2: Workload("medium", 4, 4, 64, 32, H=32, Hkv=8, d=128, layers=1, steps=5, k_scale=2.0),
    3: Workload("driving", 4, 4, 180, 256, H=32, Hkv=8, d=128, layers=36, steps=20),
    4: Workload("wide", 7, 8, 256, 512, H=32, Hkv=8, d=128, layers=1, steps=10,
                outlier_frac=0.01, outlier_scale=8.0),
    5: Workload("verify", 4, 4, 64, 32, H=32, Hkv=8, d=128, layers=1, steps=1, k_scale=2.0,
                verify_calls=64, verify_tokens=8, cache_from=2),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + rounding) >> np.uint32(16)).astype(np.uint16)


def _rng(workload: int, layer: int, step: int, tensor: int, call: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([workload, layer, step, tensor, call])))


def draw_bf16(workload: int, layer: int, step: int, tensor: int, call: int,
              shape: tuple, scale: float = 1.0) -> np.ndarray:
    x = _rng(workload, layer, step, tensor, call).standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        x = x * np.float32(scale)
    return f32_to_bf16_bits(x)


def draw_k(wid: int, wl: Workload, layer: int, step: int, call: int, n: int) -> np.ndarray:
    """K draw with the workload's structure: a global scale and/or outlier rows.

    An outlier "row" is one (token, kv-head) vector; round(frac * n * Hkv) of
    them, chosen without replacement, are multiplied by ``outlier_scale``.
    """
    x = _rng(wid, layer, step, K_ID, call).standard_normal((n, wl.Hkv, wl.d), dtype=np.float32)
    if wl.k_scale != 1.0:
        x = x * np.float32(wl.k_scale)
    if wl.outlier_frac > 0.0:
        rows = int(round(wl.outlier_frac * n * wl.Hkv))
        pick = _rng(wid, layer, step, OUTLIER_ID, call).choice(n * wl.Hkv, size=rows, replace=False)
        flat = x.reshape(n * wl.Hkv, wl.d)
        flat[pick] *= np.float32(wl.outlier_scale)
    return f32_to_bf16_bits(x)


def window_inputs(wid: int, layer: int, step: int) -> dict:
    """Q [N, H, d], K [N, Hkv, d], V [N, Hkv, d] as bf16 bits for one layer and step.

    N = window length at step 0 (prefill), else views*tok_per_frame + text_len.
    Token order: view 0's tokens, view 1's, ..., then text (for the prefill,
    each view's frames oldest first).
    """
    wl = WORKLOADS[wid]
    src = wl.cache_from if wl.cache_from is not None else wid
    swl = WORKLOADS[src]
    n = wl.tokens(step)
    return dict(
        Q=draw_bf16(src, layer, step, Q_ID, 0, (n, wl.H, wl.d)),
        K=draw_k(src, swl, layer, step, 0, n),
        V=draw_bf16(src, layer, step, V_ID, 0, (n, wl.Hkv, wl.d)),
    )


def verify_inputs(wid: int, call: int, layer: int = 0) -> dict:
    """A drafted block: Q_x [n_x, H, d], K_x / V_x [n_x, Hkv, d], fresh per call, ~N(0,1)."""
    wl = WORKLOADS[wid]
    nx = wl.verify_tokens
    step = wl.steps + 1
    return dict(
        Q=draw_bf16(wid, layer, step, Q_ID, call + 1, (nx, wl.H, wl.d)),
        K=draw_bf16(wid, layer, step, K_ID, call + 1, (nx, wl.Hkv, wl.d)),
        V=draw_bf16(wid, layer, step, V_ID, call + 1, (nx, wl.Hkv, wl.d)),
    )


# Head layout of the vision encoder's attention (the pages give none): 16 heads
# of 64, multi-head (no grouping), a ViT-style encoder layer.
FRAME_HEADS = dict(H=16, Hkv=16, d=64)


def frame_inputs(wid: int, layer: int, step: int, H: int = FRAME_HEADS["H"], Hkv: int = FRAME_HEADS["Hkv"],
                 d: int = FRAME_HEADS["d"]) -> dict:
    """The newest frame of every view, as the encoder's attention sees it:
    Q [views*n, H, d], K and V [views*n, Hkv, d] bf16 bits, ~N(0,1), token t of
    view v at row v*n + t (n = the workload's tokens per frame)."""
    wl = WORKLOADS[wid]
    rows = wl.views * wl.tok_per_frame
    return dict(
        Q=draw_bf16(wid, layer, step, FRAME_Q_ID, 0, (rows, H, d)),
        K=draw_bf16(wid, layer, step, FRAME_K_ID, 0, (rows, Hkv, d)),
        V=draw_bf16(wid, layer, step, FRAME_V_ID, 0, (rows, Hkv, d)),
    )


def hidden_inputs(wid: int, layer: int, step: int, d_model: int) -> np.ndarray:
    """Hidden states X [tokens(step), d_model] as bf16 bits, ~N(0,1), in the
    window's token order (as ``window_inputs``)."""
    wl = WORKLOADS[wid]
    return draw_bf16(wid, layer, step, X_ID, 0, (wl.tokens(step), d_model))


def proj_weight(wid: int, layer: int, d_model: int) -> np.ndarray:
    """Stacked K/V projection weight W [2*Hkv*d, d_model] as bf16 bits, drawn
    ~N(0, 1/d_model) so that X W^T is ~N(0, 1) (rows 0 .. Hkv*d-1 give K)."""
    wl = WORKLOADS[wid]
    return draw_bf16(wid, layer, 0, W_ID, 0, (2 * wl.Hkv * wl.d, d_model), scale=float(d_model) ** -0.5)
