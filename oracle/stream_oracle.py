"""Plain fp64 CPU oracle for streaming KV-cache attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links
this module. The only callers are the test suite (``tests/``), the
``smoke()`` check in ``__graft_entry__.py`` and the CPU-baseline / reference
legs of ``bench.py``. It shares no code with the CUDA library: it never
imports ``streaming_kv_cache_stream_b200`` and that package never imports it.
Both sides are fed the same seeded bf16 bytes by the input generator, which
holds none of the method's arithmetic.

What it computes, and where the pages define it (FlashDrive, arXiv 2608.12932):

* Streaming reuse of each frame's KV cache across windows, so a new window
  only adds its latest frame -- FlashDrive README (z-lab/flashdrive), list of
  techniques, "Streaming inference"; FlashDrive paper review
  (romaanj.github.io), Figure 2 caption.
* View-major token layout: all frames of camera 0, then camera 1, ...; a new
  frame goes at the end of its own view's run of tokens, not at the global end,
  and the streaming mask keeps causality across views -- FlashDrive technical
  summary (gist.science), Methodology 1, "Token Layout".
* Keys are kept pre-RoPE and rotated on the fly at the positions they hold in
  the shifted window -- FlashDrive technical summary (gist.science),
  Methodology 1, "Positional Encoding"; paper review (romaanj.github.io),
  section "Method".
* The first call of a stream only fills the cache (prefill) -- FlashDrive
  README (z-lab/flashdrive), section "Library".
* Speculative verification of a drafted 8-token block in one forward --
  FlashDrive README (z-lab/flashdrive), "Speculative reasoning (DFlash)";
  technical summary (gist.science), Methodology 2.
* Encode only the newest frame: a window step runs the vision encoder on each
  view's newest frame and reuses the rest -- technical summary (gist.science),
  Methodology 1, "Algorithmic Shortcut"; paper review (romaanj.github.io),
  Figure 2 caption. Within the encoder, a frame's tokens attend to each other
  (reading: plain bidirectional softmax attention per view, no positional
  rotation, 1/sqrt(d); the pages name no encoder internals).
* Fused projections: the Q, K, V projections are merged into one kernel --
  README (z-lab/flashdrive), "System optimizations"; technical summary,
  System Optimizations, "Kernel Fusion". Here the K/V projection of a step's
  hidden states is K = X W_k^T, V = X W_v^T, each output rounded once to bf16
  (round to nearest, ties to even) before it is cached (reading: the cache
  holds bf16, the pages give no other precision).
* Accepted draft tokens become context for the next drafted block (the
  decode stage produces reasoning tokens after the prompt; the drafter's
  blocks of 8 are accepted 5.6 tokens at a time on average) -- technical
  summary (gist.science), Methodology 2, "Efficiency".

The pages fix no RoPE variant, base, mask formula or head grouping. The
readings used here (each one also listed in the design notes):

* RoPE is rotate-half with base 10000 on 1-D integer positions: pair
  (i, i + d/2) is rotated by the angle p * base**(-2 i / d).
* A token's position is its index in the current view-major window (0 for
  the oldest frame of view 0 in every window). Only position differences
  enter the scores, so any constant offset gives the same output.
* Query p sees key q iff pos(q) <= pos(p) in the current view-major layout.
* Text tokens sit after all views, are re-supplied every step, and are among
  the queries of every step.
* Query head h reads kv head h // (H / Hkv) (contiguous grouping).
* Softmax scale 1/sqrt(d); no soft-capping, no sinks.
* Accepted tokens are appended to a decode tail right after the text (tail
  token j at position L + j); a verify block's n_x tokens sit after the tail,
  at L + tail .. L + tail + n_x - 1, see the whole window, the tail and,
  causally, each other, and are not kept. A window step starts a new window
  and with it an empty tail (a new prompt, a new reasoning pass).

Data structure: a deque of frames per view, with an insertion counter as the
frame id. This is deliberately not a ring buffer, so it shares no index
arithmetic with the device path.

Parity status: every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (brute force, library special cases, invariants,
closed-form counts, planted mistakes), except the absolute origin of the
positions, which no test can pin because the output is invariant to it
("parity unpinned" for the position origin only).
"""
from __future__ import annotations

import math
from collections import deque
from dataclasses import dataclass

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "rope_frequencies",
    "rope_rotate",
    "masked_attention",
    "ViewMajorWindow",
    "StreamOracle",
    "visible_mask",
    "kv_head_of",
    "score_scale",
    "frame_attention",
    "bf16_round",
    "project_kv",
]


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns (uint16) to float64.

    A bf16 value is the top half of an IEEE float32, so shifting the 16 bits
    up and reinterpreting gives the float32 exactly, and float32 -> float64 is
    exact too.
    """
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def rope_frequencies(d: int, base: float) -> np.ndarray:
    """Rotation frequency of each of the d/2 pairs: theta_i = base ** (-2 i / d).

    Rotate-half RoPE, base 10000 by default (reading of "Standard RoPE",
    FlashDrive technical summary (gist.science), Methodology 1, "Positional
    Encoding").
    """
    if d % 2:
        raise ValueError("head dim must be even")
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d)


def rope_rotate(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotate-half RoPE of ``x`` [N, heads, d] at integer positions ``pos`` [N].

    For pair (i, i + d/2) with angle a = pos * theta_i:
        x'_i       = x_i cos a - x_{i+d/2} sin a
        x'_{i+d/2} = x_{i+d/2} cos a + x_i sin a
    Everything in float64; cos and sin come from numpy.
    """
    x = np.asarray(x, dtype=np.float64)
    n, _, d = x.shape
    half = d // 2
    theta = rope_frequencies(d, base)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]  # [N, d/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    lo, hi = x[..., :half], x[..., half:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


def kv_head_of(h: int, H: int, Hkv: int) -> int:
    """GQA grouping: query head h reads kv head h // (H / Hkv) (contiguous groups).

    The pages name no grouping; contiguous groups is the reading taken.
    """
    return h // (H // Hkv)


def score_scale(d: int) -> float:
    """Softmax temperature 1/sqrt(d) (no soft-capping; the pages name none)."""
    return 1.0 / math.sqrt(d)


def visible_mask(qpos: np.ndarray, kpos: np.ndarray) -> np.ndarray:
    """Streaming mask: query p sees key q iff pos(q) <= pos(p).

    Causality over the current view-major layout (FlashDrive technical summary
    (gist.science), Methodology 1, "Token Layout": the streaming mask keeps
    cross-view causality).
    """
    return np.asarray(kpos)[None, :] <= np.asarray(qpos)[:, None]


def masked_attention(Q: np.ndarray, qpos: np.ndarray, K: np.ndarray, V: np.ndarray,
                     kpos: np.ndarray, base: float) -> np.ndarray:
    """Dense attention of pre-RoPE queries against pre-RoPE keys, in float64.

    Q [Nq, H, d], K and V [Nk, Hkv, d], positions qpos [Nq], kpos [Nk].
    Rotates Q and K at their positions (V is not rotated), scores each query
    head h against kv head h // (H/Hkv) scaled by 1/sqrt(d), applies the
    streaming mask, and normalises with a softmax. Returns [Nq, H, d].
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    nq, H, d = Q.shape
    Hkv = K.shape[1]
    if H % Hkv:
        raise ValueError("H must be a multiple of Hkv")
    q_rot = rope_rotate(Q, qpos, base)
    k_rot = rope_rotate(K, kpos, base)
    mask = visible_mask(qpos, kpos)
    if not mask.any(axis=1).all():
        raise ValueError("a query row sees no key")
    out = np.empty((nq, H, d), dtype=np.float64)
    scale = score_scale(d)
    for h in range(H):
        kv = kv_head_of(h, H, Hkv)
        s = (q_rot[:, h, :] @ k_rot[:, kv, :].T) * scale
        s = np.where(mask, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ V[:, kv, :]
    return out


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (8 significant bits), ties
    to even, directly (no intermediate float32 rounding). Finite inputs within
    the bf16 range; returns float64."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    e = np.floor(np.log2(np.abs(x[nz])))
    e = np.maximum(e, -126.0)  # below the smallest normal the spacing stays 2^-133
    ulp = np.exp2(e - 7.0)
    out[nz] = np.rint(x[nz] / ulp) * ulp  # rint: nearest, ties to even
    return out


def project_kv(X: np.ndarray, W: np.ndarray, Hkv: int, d: int):
    """K/V projection of hidden states: X [N, d_model] (bf16 values as float64),
    W [2*Hkv*d, d_model] (rows 0 .. Hkv*d-1 project K, the rest V, as in a
    linear layer's weight). Returns K, V [N, Hkv, d]: X W^T in float64, each
    element rounded once to bf16."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    if W.shape != (2 * Hkv * d, X.shape[1]):
        raise ValueError("W must be [2*Hkv*d, d_model]")
    Y = bf16_round(X @ W.T)
    n = X.shape[0]
    return Y[:, :Hkv * d].reshape(n, Hkv, d), Y[:, Hkv * d:].reshape(n, Hkv, d)


def frame_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, views: int, n: int) -> np.ndarray:
    """Encoder attention over the newest frame of each view, in float64.

    Q [views*n, H, d], K and V [views*n, Hkv, d], tokens view-major (view v's
    frame is rows v*n .. v*n + n - 1). Every token of view v attends to every
    token of view v's frame (bidirectional, no mask inside the frame) and to
    nothing else; no rotation; scores scaled by 1/sqrt(d); query head h reads
    kv head h // (H/Hkv). Returns [views*n, H, d].
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    nt, H, d = Q.shape
    Hkv = K.shape[1]
    if nt != views * n or K.shape[0] != nt or V.shape[0] != nt or H % Hkv:
        raise ValueError("bad frame shapes")
    out = np.empty((nt, H, d), dtype=np.float64)
    scale = score_scale(d)
    for v in range(views):
        rows = slice(v * n, (v + 1) * n)
        for h in range(H):
            kv = kv_head_of(h, H, Hkv)
            s = (Q[rows, h, :] @ K[rows, kv, :].T) * scale
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[rows, h, :] = p @ V[rows, kv, :]
    return out


@dataclass
class _Frame:
    frame_id: int
    K: np.ndarray  # [n, Hkv, d] float64, pre-RoPE
    V: np.ndarray


class ViewMajorWindow:
    """The sliding window of T frames per view, kept as one deque per view.

    Prefill pushes T frames per view. A window step appends each view's new
    frame at the right of that view's deque and drops the oldest frame at the
    left ("new tokens are inserted at the end of each view's sequence rather
    than appended globally", FlashDrive technical summary (gist.science),
    Methodology 1, "Token Layout"; the window slides by one frame, same page,
    Problem Statement, item 1). Text K/V is replaced by the fresh text of
    each step.
    """

    def __init__(self, views: int, frames: int, tok_per_frame: int, text_len: int):
        if min(views, frames, tok_per_frame) < 1 or text_len < 0:
            raise ValueError("bad window shape")
        self.V, self.T, self.n, self.X = views, frames, tok_per_frame, text_len
        self.views: list[deque] = [deque() for _ in range(views)]
        self.text_K = None
        self.text_V = None
        self.next_id = [0] * views
        self.filled = False
        self.tail_K: list = []  # accepted decode tokens after the text, oldest first
        self.tail_V: list = []

    @property
    def window_len(self) -> int:
        return self.V * self.T * self.n + self.X

    @property
    def step_tokens(self) -> int:
        return self.V * self.n + self.X

    def _push(self, v: int, K: np.ndarray, V: np.ndarray) -> None:
        self.views[v].append(_Frame(self.next_id[v], K.copy(), V.copy()))
        self.next_id[v] += 1

    def prefill(self, K: np.ndarray, V: np.ndarray) -> None:
        """K, V [L, Hkv, d] in window order: view 0's T frames oldest first, ..., then text."""
        if K.shape[0] != self.window_len or V.shape[0] != self.window_len:
            raise ValueError("prefill needs the whole window")
        for dq in self.views:
            dq.clear()
        self.next_id = [0] * self.V
        for v in range(self.V):
            for f in range(self.T):
                a = (v * self.T + f) * self.n
                self._push(v, K[a:a + self.n], V[a:a + self.n])
        t0 = self.V * self.T * self.n
        self.text_K, self.text_V = K[t0:].copy(), V[t0:].copy()
        self.tail_K, self.tail_V = [], []
        self.filled = True

    def step(self, K_new: np.ndarray, V_new: np.ndarray) -> None:
        """K_new, V_new [V*n + X, Hkv, d]: view 0's new frame, view 1's, ..., then text."""
        if not self.filled:
            raise ValueError("step before prefill")
        if K_new.shape[0] != self.step_tokens or V_new.shape[0] != self.step_tokens:
            raise ValueError("a step inserts one frame per view plus the text")
        for v in range(self.V):
            a = v * self.n
            self._push(v, K_new[a:a + self.n], V_new[a:a + self.n])
            self.views[v].popleft()
        t0 = self.V * self.n
        self.text_K, self.text_V = K_new[t0:].copy(), V_new[t0:].copy()
        self.tail_K, self.tail_V = [], []

    def append(self, K_acc: np.ndarray, V_acc: np.ndarray) -> None:
        """Accepted decode tokens [n, Hkv, d], appended after the text (and the earlier tail)."""
        if not self.filled:
            raise ValueError("append before prefill")
        for i in range(K_acc.shape[0]):
            self.tail_K.append(np.array(K_acc[i], dtype=np.float64))
            self.tail_V.append(np.array(V_acc[i], dtype=np.float64))

    @property
    def tail_len(self) -> int:
        return len(self.tail_K)

    def materialise_tail(self, Hkv: int, d: int):
        """Tail K, V [tail, Hkv, d] (empty arrays when there is none)."""
        if not self.tail_K:
            z = np.zeros((0, Hkv, d))
            return z, z.copy()
        return np.stack(self.tail_K), np.stack(self.tail_V)

    def materialise(self):
        """Window K, V [L, Hkv, d] in view-major order, plus per-row bookkeeping.

        Returns (K, V, view, frame_id, token) where view/frame_id/token are -1
        for text rows (token holds the text index there).
        """
        ks, vs, view, fid, tok = [], [], [], [], []
        for v, dq in enumerate(self.views):
            for fr in dq:
                ks.append(fr.K)
                vs.append(fr.V)
                view += [v] * self.n
                fid += [fr.frame_id] * self.n
                tok += list(range(self.n))
        ks.append(self.text_K)
        vs.append(self.text_V)
        view += [-1] * self.X
        fid += [-1] * self.X
        tok += list(range(self.X))
        return (np.concatenate(ks, axis=0), np.concatenate(vs, axis=0),
                np.array(view), np.array(fid), np.array(tok))

    def key_positions(self) -> np.ndarray:
        """Every window token's position is its index in the current window."""
        return np.arange(self.window_len, dtype=np.int64)

    def step_query_positions(self) -> np.ndarray:
        """Positions of a step's queries: each view's newest frame, then the text.

        View v's newest frame is the last of that view's T frames, so its
        token i sits at v*T*n + (T-1)*n + i; text token j sits at V*T*n + j.
        """
        pos = []
        for v in range(self.V):
            start = v * self.T * self.n + (self.T - 1) * self.n
            pos += list(range(start, start + self.n))
        pos += list(range(self.V * self.T * self.n, self.window_len))
        return np.array(pos, dtype=np.int64)


class StreamOracle:
    """One layer's streaming attention: window bookkeeping plus dense attention.

    ``prefill`` is the stream's first call (whole window, full causal over the
    view-major sequence); ``step`` is a window step (new frame per view plus
    text); ``append`` persists accepted decode tokens after the text;
    ``verify`` attends a drafted block after the text and the tail without
    keeping it.
    Inputs are float64 arrays (use ``bf16_bits_to_f64`` on the shared bf16
    bytes). ``rows`` restricts the computed queries to a subset of query
    indices, so full-size cases can be checked on samples.
    """

    def __init__(self, views, frames, tok_per_frame, text_len, H, Hkv, d, rope_base=10000.0):
        if H % Hkv:
            raise ValueError("H must be a multiple of Hkv")
        self.win = ViewMajorWindow(views, frames, tok_per_frame, text_len)
        self.H, self.Hkv, self.d, self.base = H, Hkv, d, float(rope_base)

    def _attend(self, Q, qpos, rows, K, V, kpos):
        if rows is not None:
            rows = np.asarray(rows)
            Q, qpos = Q[rows], qpos[rows]
        return masked_attention(Q, qpos, K, V, kpos, self.base)

    def prefill(self, Q, K, V, rows=None):
        self.win.prefill(K, V)
        Kw, Vw, *_ = self.win.materialise()
        pos = self.win.key_positions()
        return self._attend(Q, pos, rows, Kw, Vw, pos)

    def step(self, Q, K_new, V_new, rows=None):
        self.win.step(K_new, V_new)
        Kw, Vw, *_ = self.win.materialise()
        return self._attend(Q, self.win.step_query_positions(), rows, Kw, Vw,
                            self.win.key_positions())

    def append(self, K_acc, V_acc):
        """Persist accepted decode tokens after the text (see ViewMajorWindow.append)."""
        self.win.append(K_acc, V_acc)

    def verify(self, Q_x, K_x, V_x, rows=None):
        """A drafted block of n_x tokens right after the text and the decode
        tail (positions L + tail .. L + tail + n_x - 1), not persisted."""
        Kw, Vw, *_ = self.win.materialise()
        Kt, Vt = self.win.materialise_tail(self.Hkv, self.d)
        L = self.win.window_len
        t = Kt.shape[0]
        nx = Q_x.shape[0]
        K = np.concatenate([Kw, Kt, K_x], axis=0)
        V = np.concatenate([Vw, Vt, V_x], axis=0)
        kpos = np.arange(L + t + nx, dtype=np.int64)
        qpos = np.arange(L + t, L + t + nx, dtype=np.int64)
        return self._attend(Q_x, qpos, rows, K, V, kpos)

    def cache_rows(self):
        """Pre-RoPE cached rows with their (view, frame_id, token, position).

        Used for the bit-exact comparison with the device cache: rows match by
        (view, frame_id, token) for frames, by text index for text (view -1)
        and by tail index for the decode tail (view -2).
        """
        Kw, Vw, view, fid, tok = self.win.materialise()
        Kt, Vt = self.win.materialise_tail(self.Hkv, self.d)
        t = Kt.shape[0]
        L = self.win.window_len
        return dict(K=np.concatenate([Kw, Kt]), V=np.concatenate([Vw, Vt]),
                    view=np.concatenate([view, np.full(t, -2)]),
                    frame_id=np.concatenate([fid, np.full(t, -1)]),
                    token=np.concatenate([tok, np.arange(t)]),
                    pos=np.arange(L + t, dtype=np.int64))
