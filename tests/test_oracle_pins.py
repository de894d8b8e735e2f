"""Pins of the fp64 CPU oracle against things other than itself (CPU only).

Each ``pin_*`` helper raises AssertionError when the oracle disagrees with:
  * brute force written from scratch with Python scalars (math.cos/sin/exp);
  * a library routine for a special case (Hugging Face Llama rotate-half RoPE;
    torch's scaled_dot_product_attention in float64, causal, GQA);
  * the complex-number form of RoPE and its group properties;
  * invariants the pages imply (relative positions only; streaming output equals
    a from-scratch causal prefill of the current window; ring contents);
  * closed-form counts (visible query-key pairs; the 1/T token fraction that
    the pages quote as "75%").
``test_planted_*`` swap a deliberately wrong piece into the oracle and check
that some pin catches it.
"""
from __future__ import annotations

import cmath
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.stream_oracle as so
from oracle import StreamOracle, ViewMajorWindow, bf16_bits_to_f64, masked_attention, rope_rotate
from streaming_kv_cache_stream_b200.inputs import WORKLOADS, f32_to_bf16_bits, verify_inputs, window_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TINY = dict(views=2, frames=2, tok_per_frame=3, text_len=2, H=2, Hkv=1, d=8)
TINY_G = dict(views=3, frames=3, tok_per_frame=2, text_len=3, H=4, Hkv=2, d=8)


def _rand(rng, *shape):
    return f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


# --------------------------------------------------------------------------- RoPE

def _rope_complex(x, pos, base):
    """RoPE as complex multiplication: z_i = x_i + 1j x_{i+d/2} times e^{1j p theta_i}."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    out = np.empty_like(x)
    for t in range(x.shape[0]):
        for h in range(x.shape[1]):
            for i in range(half):
                theta = math.exp(-(2.0 * i / d) * math.log(base))
                z = complex(x[t, h, i], x[t, h, i + half]) * cmath.exp(1j * pos[t] * theta)
                out[t, h, i], out[t, h, i + half] = z.real, z.imag
    return out


def pin_rope_complex_form(base=10000.0):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 3, 16))
    pos = np.array([0, 1, 2, 5, 100, 1057, 14847])
    np.testing.assert_allclose(rope_rotate(x, pos, base), _rope_complex(x, pos, base), rtol=0, atol=1e-9)


def pin_rope_matches_hf_llama(d=64, base=10000.0):
    """Hugging Face Llama RoPE (rotate-half, inv_freq = base^(-2i/d)) at small positions."""
    from transformers import LlamaConfig
    from transformers.models.llama import modeling_llama as m

    cfg = LlamaConfig(hidden_size=2 * d, num_attention_heads=2, num_key_value_heads=1, head_dim=d,
                      rope_theta=base, max_position_embeddings=4096)
    emb = m.LlamaRotaryEmbedding(cfg)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((9, 2, d))
    pos = np.array([0, 1, 2, 3, 7, 11, 16, 31, 63])
    xt = torch.tensor(x).permute(1, 0, 2)[None]  # [1, heads, N, d]
    cos, sin = emb(xt, torch.tensor(pos)[None])
    q_hf, _ = m.apply_rotary_pos_emb(xt, xt, cos, sin)
    ref = q_hf[0].permute(1, 0, 2).numpy()
    # HF builds its angles in float32, hence the loose tolerance; the convention
    # (pairing, direction, frequencies) is what this pins.
    np.testing.assert_allclose(rope_rotate(x, pos, base), ref, rtol=0, atol=2e-4)


def pin_rope_group_properties(base=10000.0):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 2, 32))
    zero = np.zeros(5, dtype=np.int64)
    np.testing.assert_array_equal(rope_rotate(x, zero, base), x)
    a = np.array([3, 17, 250, 1000, 9999])
    b = np.array([5, 1, 33, 2000, 1])
    np.testing.assert_allclose(rope_rotate(rope_rotate(x, a, base), b, base), rope_rotate(x, a + b, base),
                               atol=1e-9)
    r = rope_rotate(x, a, base)
    half = 16
    np.testing.assert_allclose(r[..., :half] ** 2 + r[..., half:] ** 2,
                               x[..., :half] ** 2 + x[..., half:] ** 2, rtol=1e-12)


def pin_rope_relative(base=10000.0):
    """<R(p) q, R(p') k> depends only on p - p'."""
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 1, 64))
    k = rng.standard_normal((1, 1, 64))
    ref = float((rope_rotate(q, np.array([40]), base) * rope_rotate(k, np.array([13]), base)).sum())
    for c in (1, 37, 10_000, 123_457):
        got = float((rope_rotate(q, np.array([40 + c]), base) * rope_rotate(k, np.array([13 + c]), base)).sum())
        assert abs(got - ref) < 1e-9, (c, got, ref)


def test_rope_complex_form():
    pin_rope_complex_form()


def test_rope_matches_hf_llama():
    pin_rope_matches_hf_llama()
    pin_rope_matches_hf_llama(d=128)


def test_rope_group_properties():
    pin_rope_group_properties()


def test_rope_relative_positions():
    pin_rope_relative()


def test_bf16_upcast_exact():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x7F7F, 0x0001], dtype=np.uint16)
    want = np.array([1.0, -2.0, 1.0078125, 0.0, -0.0, 3.3895313892515355e38, 9.183549615799121e-41])
    np.testing.assert_array_equal(bf16_bits_to_f64(bits), want)
    # round-to-nearest-even of the generator, ties included
    f = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9], dtype=np.float32)
    np.testing.assert_array_equal(f32_to_bf16_bits(f), np.array([0x3F80, 0x3F82, 0x3F80], dtype=np.uint16))


# ------------------------------------------------------------ brute force (tiny)

class _History:
    """Every frame ever seen per view; the window is rebuilt from the last T each step."""

    def __init__(self, views, frames, tok_per_frame, text_len, **_):
        self.V, self.T, self.n, self.X = views, frames, tok_per_frame, text_len
        self.frames = [[] for _ in range(views)]
        self.text = None

    def prefill(self, K, V):
        for v in range(self.V):
            for f in range(self.T):
                a = (v * self.T + f) * self.n
                self.frames[v].append((K[a:a + self.n], V[a:a + self.n]))
        t = self.V * self.T * self.n
        self.text = (K[t:], V[t:])

    def step(self, K, V):
        for v in range(self.V):
            self.frames[v].append((K[v * self.n:(v + 1) * self.n], V[v * self.n:(v + 1) * self.n]))
        t = self.V * self.n
        self.text = (K[t:], V[t:])
        self.tail = []

    def append(self, K, V):
        self.tail = getattr(self, "tail", []) + [(K[i], V[i]) for i in range(K.shape[0])]

    def window(self):
        toks = []
        for v in range(self.V):
            for Kf, Vf in self.frames[v][-self.T:]:
                for i in range(self.n):
                    toks.append((Kf[i], Vf[i]))
        for j in range(self.X):
            toks.append((self.text[0][j], self.text[1][j]))
        return toks


def _brute_rot(vec, p, base):
    d = len(vec)
    half = d // 2
    out = [0.0] * d
    for i in range(half):
        th = base ** (-(2.0 * i) / d)
        c, s = math.cos(p * th), math.sin(p * th)
        out[i] = vec[i] * c - vec[i + half] * s
        out[i + half] = vec[i + half] * c + vec[i] * s
    return out


def _brute_attend(qs, qpos, toks, H, Hkv, d, base=10000.0):
    """Scalar Python: every score, mask, exp and sum written out."""
    G = H // Hkv
    out = np.zeros((len(qs), H, d))
    for a, (qv, p) in enumerate(zip(qs, qpos)):
        for h in range(H):
            kv = h // G
            qr = _brute_rot([float(x) for x in qv[h]], p, base)
            scores, vals = [], []
            for kpos, (kvec, vvec) in enumerate(toks):
                if kpos > p:
                    continue
                kr = _brute_rot([float(x) for x in kvec[kv]], kpos, base)
                scores.append(sum(qr[i] * kr[i] for i in range(d)) / math.sqrt(d))
                vals.append(vvec[kv])
            mx = max(scores)
            w = [math.exp(s - mx) for s in scores]
            tot = sum(w)
            for i in range(d):
                out[a, h, i] = sum(w[j] * float(vals[j][i]) for j in range(len(w))) / tot
    return out


def _step_qpos_brute(V, T, n, X):
    pos = []
    for v in range(V):
        pos += [v * T * n + (T - 1) * n + i for i in range(n)]
    pos += [V * T * n + j for j in range(X)]
    return pos


def pin_brute_force(shape, steps=3, seed=5):
    rng = np.random.default_rng(seed)
    V, T, n, X, H, Hkv, d = (shape[k] for k in ("views", "frames", "tok_per_frame", "text_len", "H", "Hkv", "d"))
    L = V * T * n + X
    orc = StreamOracle(V, T, n, X, H, Hkv, d)
    hist = _History(**shape)
    Q = bf16_bits_to_f64(_rand(rng, L, H, d))
    K = bf16_bits_to_f64(_rand(rng, L, Hkv, d))
    Vv = bf16_bits_to_f64(_rand(rng, L, Hkv, d))
    got = orc.prefill(Q, K, Vv)
    hist.prefill(K, Vv)
    want = _brute_attend(list(Q), list(range(L)), hist.window(), H, Hkv, d)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    N = V * n + X
    for _ in range(steps):
        Q = bf16_bits_to_f64(_rand(rng, N, H, d))
        K = bf16_bits_to_f64(_rand(rng, N, Hkv, d))
        Vv = bf16_bits_to_f64(_rand(rng, N, Hkv, d))
        got = orc.step(Q, K, Vv)
        hist.step(K, Vv)
        want = _brute_attend(list(Q), _step_qpos_brute(V, T, n, X), hist.window(), H, Hkv, d)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def pin_brute_force_decode_tail(shape, seed=9):
    """Drafted blocks verified against window + accepted tail, rebuilt from the
    full history with scalar loops: tail tokens follow the text, a block follows
    the tail, and a window step empties the tail."""
    rng = np.random.default_rng(seed)
    V, T, n, X, H, Hkv, d = (shape[k] for k in ("views", "frames", "tok_per_frame", "text_len", "H", "Hkv", "d"))
    L = V * T * n + X
    N = V * n + X
    orc = StreamOracle(V, T, n, X, H, Hkv, d)
    hist = _History(**shape)

    def draw(m, heads):
        return bf16_bits_to_f64(_rand(rng, m, heads, d))

    K, Vv = draw(L, Hkv), draw(L, Hkv)
    orc.prefill(draw(L, H), K, Vv)
    hist.prefill(K, Vv)
    hist.tail = []
    for rnd in range(2):
        for n_acc, n_x in ((3, 2), (2, 3)):
            Qx, Kx, Vx = draw(n_x, H), draw(n_x, Hkv), draw(n_x, Hkv)
            got = orc.verify(Qx, Kx, Vx)
            toks = hist.window() + hist.tail + [(Kx[i], Vx[i]) for i in range(n_x)]
            t = len(hist.tail)
            want = _brute_attend(list(Qx), [L + t + j for j in range(n_x)], toks, H, Hkv, d)
            np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
            Ka, Va = draw(n_acc, Hkv), draw(n_acc, Hkv)
            orc.append(Ka, Va)
            hist.append(Ka, Va)
        # a window step: new frames, new text, no tail
        K, Vv = draw(N, Hkv), draw(N, Hkv)
        orc.step(draw(N, H), K, Vv)
        hist.step(K, Vv)


def test_brute_force_tiny():
    pin_brute_force(TINY, steps=3)


def test_brute_force_decode_tail():
    pin_brute_force_decode_tail(TINY)
    pin_brute_force_decode_tail(TINY_G, seed=10)


def test_append_then_verify_equals_longer_block():
    """Appending accepted tokens, then verifying a block, gives the block's rows
    of one verify over (accepted ++ block): the tail sits exactly where the
    accepted tokens sat in the longer block."""
    wl = WORKLOADS[1]
    rng = np.random.default_rng(12)
    a = StreamOracle(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d)
    b = StreamOracle(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d)
    inp = window_inputs(1, 0, 0)
    f = [bf16_bits_to_f64(inp[k]) for k in ("Q", "K", "V")]
    a.prefill(*f)
    b.prefill(*f)
    n_acc, nx = 5, 8
    Q = bf16_bits_to_f64(_rand(rng, n_acc + nx, wl.H, wl.d))
    K = bf16_bits_to_f64(_rand(rng, n_acc + nx, wl.Hkv, wl.d))
    Vv = bf16_bits_to_f64(_rand(rng, n_acc + nx, wl.Hkv, wl.d))
    long = a.verify(Q, K, Vv)
    b.append(K[:n_acc], Vv[:n_acc])
    short = b.verify(Q[n_acc:], K[n_acc:], Vv[n_acc:])
    np.testing.assert_allclose(short, long[n_acc:], rtol=0, atol=1e-13)
    assert b.cache_rows()["K"].shape[0] == wl.window_len + n_acc


def test_brute_force_tiny_gqa():
    pin_brute_force(TINY_G, steps=4)


# ----------------------------------------------- library special case: first window

def _sdpa_causal(Q, K, V, H, Hkv, base):
    """Float64 torch SDPA, causal, GQA, on keys/queries rotated by the complex form."""
    L = Q.shape[0]
    pos = np.arange(L)
    qr = torch.tensor(_rope_complex(Q, pos, base)).permute(1, 0, 2)[None]
    kr = torch.tensor(_rope_complex(K, pos, base)).permute(1, 0, 2)[None]
    vv = torch.tensor(V).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qr, kr, vv, is_causal=True, enable_gqa=(H != Hkv))
    return o[0].permute(1, 0, 2).numpy()


def pin_first_window_is_causal_sdpa(wid=1):
    wl = WORKLOADS[wid]
    inp = window_inputs(wid, 0, 0)
    Q, K, V = (bf16_bits_to_f64(inp[k]) for k in ("Q", "K", "V"))
    orc = StreamOracle(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d)
    got = orc.prefill(Q, K, V)
    want = _sdpa_causal(Q, K, V, wl.H, wl.Hkv, wl.rope_base)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)


def test_first_window_is_causal_sdpa():
    pin_first_window_is_causal_sdpa(1)


# ------------------------------------ streaming == from-scratch prefill of the window

def pin_step_equals_rescratch(shape, steps=3, seed=7):
    """After every step, the step's outputs are rows of a fresh causal prefill
    (torch SDPA) over the window rebuilt from the full history."""
    rng = np.random.default_rng(seed)
    V, T, n, X, H, Hkv, d = (shape[k] for k in ("views", "frames", "tok_per_frame", "text_len", "H", "Hkv", "d"))
    L = V * T * n + X
    N = V * n + X
    orc = StreamOracle(V, T, n, X, H, Hkv, d)
    hist = _History(**shape)
    K = bf16_bits_to_f64(_rand(rng, L, Hkv, d))
    Vv = bf16_bits_to_f64(_rand(rng, L, Hkv, d))
    orc.prefill(bf16_bits_to_f64(_rand(rng, L, H, d)), K, Vv)
    hist.prefill(K, Vv)
    qpos = np.array(_step_qpos_brute(V, T, n, X))
    for _ in range(steps):
        Q = bf16_bits_to_f64(_rand(rng, N, H, d))
        K = bf16_bits_to_f64(_rand(rng, N, Hkv, d))
        Vv = bf16_bits_to_f64(_rand(rng, N, Hkv, d))
        got = orc.step(Q, K, Vv)
        hist.step(K, Vv)
        toks = hist.window()
        Kw = np.stack([t[0] for t in toks])
        Vw = np.stack([t[1] for t in toks])
        Qfull = bf16_bits_to_f64(_rand(rng, L, H, d))
        Qfull[qpos] = Q
        want = _sdpa_causal(Qfull, Kw, Vw, H, Hkv, 10000.0)[qpos]
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)


def test_step_equals_rescratch():
    pin_step_equals_rescratch(dict(views=3, frames=4, tok_per_frame=5, text_len=4, H=4, Hkv=2, d=16), steps=6)


def test_verify_equals_causal_tail():
    """The verify block is the last n_x rows of a causal prefill over window + block."""
    wl = WORKLOADS[1]
    rng = np.random.default_rng(11)
    orc = StreamOracle(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d)
    inp = window_inputs(1, 0, 0)
    orc.prefill(*(bf16_bits_to_f64(inp[k]) for k in ("Q", "K", "V")))
    nx = 8
    Qx = bf16_bits_to_f64(_rand(rng, nx, wl.H, wl.d))
    Kx = bf16_bits_to_f64(_rand(rng, nx, wl.Hkv, wl.d))
    Vx = bf16_bits_to_f64(_rand(rng, nx, wl.Hkv, wl.d))
    got = orc.verify(Qx, Kx, Vx)
    c = orc.cache_rows()
    L = wl.window_len
    Qf = np.concatenate([bf16_bits_to_f64(_rand(rng, L, wl.H, wl.d)), Qx])
    want = _sdpa_causal(Qf, np.concatenate([c["K"], Kx]), np.concatenate([c["V"], Vx]), wl.H, wl.Hkv, 10000.0)[L:]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)
    # not persisted: the window is unchanged
    np.testing.assert_array_equal(orc.cache_rows()["K"], c["K"])


# ---------------------------------------------------- relative-position invariance

def pin_shift_invariance(wid=1):
    wl = WORKLOADS[wid]
    inp = window_inputs(wid, 0, 0)
    Q, K, V = (bf16_bits_to_f64(inp[k]) for k in ("Q", "K", "V"))
    pos = np.arange(wl.window_len)
    ref = masked_attention(Q, pos, K, V, pos, wl.rope_base)
    for c in (1, 37, 10_000):
        got = masked_attention(Q, pos + c, K, V, pos + c, wl.rope_base)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-9)


def test_shift_invariance():
    pin_shift_invariance(1)


# --------------------------------------------------------------- ring invariants

def test_window_frame_ids_and_eviction():
    T = 4
    w = ViewMajorWindow(views=3, frames=T, tok_per_frame=2, text_len=1)
    L = w.window_len
    z = np.zeros((L, 1, 2))
    w.prefill(z, z)
    for k in range(1, 2 * T + 2):
        zz = np.zeros((w.step_tokens, 1, 2))
        w.step(zz, zz)
        _, _, view, fid, _ = w.materialise()
        for v in range(3):
            ids = sorted(set(fid[view == v].tolist()))
            assert ids == list(range(k, k + T)), (k, v, ids)
        if k >= T:  # every prefill frame is gone after T steps
            assert fid[view >= 0].min() >= T
        np.testing.assert_array_equal(w.key_positions(), np.arange(L))


def test_new_frame_fraction_is_one_over_T():
    """The pages' 75% (4-frame window): a step recomputes 1 of every T frame tokens."""
    with open(os.path.join(GOLDEN, "paper_numbers.json")) as f:
        g = json.load(f)
    T = g["window_frames"]
    for wid in (2, 3):
        wl = WORKLOADS[wid]
        assert wl.frames == T
        w = ViewMajorWindow(wl.views, wl.frames, wl.tok_per_frame, wl.text_len)
        new_frame_tokens = int((w.step_query_positions() < wl.views * T * wl.tok_per_frame).sum())
        window_frame_tokens = wl.views * T * wl.tok_per_frame
        assert 1.0 - new_frame_tokens / window_frame_tokens == pytest.approx(g["effective_sequence_reduction"])


# ------------------------------------------------------------- closed-form counts

def closed_form_step_pairs(V, T, n, X):
    """Visible (query, key) pairs of one window step, summed in closed form.

    View v's new-frame token i sits at v*T*n + (T-1)*n + i and sees that many
    keys plus one; text token j sees V*T*n + j + 1 keys.
    """
    frames = V * n * ((T - 1) * n + 1) + T * n * n * V * (V - 1) // 2 + V * n * (n - 1) // 2
    text = X * (V * T * n + 1) + X * (X - 1) // 2
    return frames + text


def test_visible_pairs_closed_form_and_golden():
    with open(os.path.join(GOLDEN, "visible_pairs.json")) as f:
        g = json.load(f)
    for wid in (1, 2, 3, 4):
        wl = WORKLOADS[wid]
        w = ViewMajorWindow(wl.views, wl.frames, wl.tok_per_frame, wl.text_len)
        dense = int(so.visible_mask(w.step_query_positions(), w.key_positions()).sum())
        cf = closed_form_step_pairs(wl.views, wl.frames, wl.tok_per_frame, wl.text_len)
        assert dense == cf == g[str(wid)]["step_pairs"], (wid, dense, cf)
        L = wl.window_len
        assert g[str(wid)]["prefill_pairs"] == L * (L + 1) // 2
    # verify block: n_x queries at L.. see L + k + 1 keys
    wl = WORKLOADS[5]
    L, nx = wl.window_len, wl.verify_tokens
    assert g["5"]["verify_pairs"] == sum(L + k + 1 for k in range(nx))


def test_mask_counts_per_query():
    V, T, n, X = 3, 4, 5, 6
    w = ViewMajorWindow(V, T, n, X)
    m = so.visible_mask(w.step_query_positions(), w.key_positions())
    for i in range(n):  # view 0's new frame token i
        assert m[i].sum() == T * n - n + i + 1
    for j in range(X):
        assert m[V * n + j].sum() == V * T * n + j + 1
    w1 = ViewMajorWindow(1, T, n, 0)  # one view, no text: plain causal over frames
    m1 = so.visible_mask(w1.step_query_positions(), w1.key_positions())
    assert np.array_equal(m1, np.tril(np.ones((T * n, T * n), bool))[(T - 1) * n:])


def test_inputs_deterministic_and_shaped():
    a = window_inputs(4, 0, 1)
    b = window_inputs(4, 0, 1)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    wl = WORKLOADS[4]
    assert a["Q"].shape == (wl.step_tokens, wl.H, wl.d)
    assert a["K"].shape == (wl.step_tokens, wl.Hkv, wl.d)
    K = bf16_bits_to_f64(a["K"]).reshape(-1, wl.d)
    big = np.abs(K).max(axis=1) > 6.0  # x8 outliers stand far out of N(0,1)
    assert abs(int(big.sum()) - round(0.01 * K.shape[0])) <= 2
    v = verify_inputs(5, 3)
    assert v["Q"].shape == (8, 32, 128)


# ------------------------------------------------------------- planted mistakes

def _expect_caught(monkeypatch, target, replacement, pins):
    monkeypatch.setattr(target[0], target[1], replacement)
    caught = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, ValueError, FloatingPointError):
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake in {target[1]}"


ALL_PINS = [
    pin_rope_complex_form,
    pin_rope_matches_hf_llama,
    pin_rope_group_properties,
    pin_rope_relative,
    lambda: pin_brute_force(TINY, steps=2),
    lambda: pin_brute_force(TINY_G, steps=2),
    pin_first_window_is_causal_sdpa,
]


def test_planted_wrong_frequency(monkeypatch):
    _expect_caught(monkeypatch, (so, "rope_frequencies"),
                   lambda d, base: np.power(float(base), -1.0 * np.arange(d // 2) / d), ALL_PINS)


def test_planted_wrong_rotation_sign(monkeypatch):
    orig = so.rope_rotate

    def bad(x, pos, base):
        return orig(x, -np.asarray(pos), base)
    _expect_caught(monkeypatch, (so, "rope_rotate"), bad, ALL_PINS)


def test_planted_interleaved_pairs(monkeypatch):
    orig = so.rope_rotate

    def bad(x, pos, base):  # GPT-J style pairing (2i, 2i+1) instead of (i, i+d/2)
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        perm = np.concatenate([np.arange(0, d, 2), np.arange(1, d, 2)])
        inv = np.argsort(perm)
        return orig(x[..., perm], pos, base)[..., inv]
    _expect_caught(monkeypatch, (so, "rope_rotate"), bad, ALL_PINS)


def test_planted_strict_mask(monkeypatch):
    _expect_caught(monkeypatch, (so, "visible_mask"),
                   lambda q, k: np.asarray(k)[None, :] < np.asarray(q)[:, None], ALL_PINS)


def test_planted_one_future_key(monkeypatch):
    _expect_caught(monkeypatch, (so, "visible_mask"),
                   lambda q, k: np.asarray(k)[None, :] <= np.asarray(q)[:, None] + 1, ALL_PINS)


def test_planted_gqa_interleaved(monkeypatch):
    _expect_caught(monkeypatch, (so, "kv_head_of"), lambda h, H, Hkv: h % Hkv, ALL_PINS)


def test_planted_missing_scale(monkeypatch):
    _expect_caught(monkeypatch, (so, "score_scale"), lambda d: 1.0, ALL_PINS)


def test_planted_newest_frame_first(monkeypatch):
    orig = ViewMajorWindow.materialise

    def bad(self):
        for dq in self.views:
            dq.reverse()
        try:
            return orig(self)
        finally:
            for dq in self.views:
                dq.reverse()
    _expect_caught(monkeypatch, (ViewMajorWindow, "materialise"), bad, ALL_PINS)


def test_planted_no_eviction(monkeypatch):
    orig = ViewMajorWindow.step

    def bad(self, K_new, V_new):  # evicts the newest frame instead of the oldest
        for v in range(self.V):
            a = v * self.n
            self.views[v].pop()
            self._push(v, K_new[a:a + self.n], V_new[a:a + self.n])
        t0 = self.V * self.n
        self.text_K, self.text_V = K_new[t0:].copy(), V_new[t0:].copy()
    _expect_caught(monkeypatch, (ViewMajorWindow, "step"), bad, ALL_PINS)


TAIL_PINS = [lambda: pin_brute_force_decode_tail(TINY), lambda: pin_brute_force_decode_tail(TINY_G, seed=10)]


def test_planted_tail_before_text(monkeypatch):
    """A tail spliced in before the text (wrong positions) is caught."""
    def bad(self, Q_x, K_x, V_x, rows=None):
        Kw, Vw, *_ = self.win.materialise()
        Kt, Vt = self.win.materialise_tail(self.Hkv, self.d)
        X = self.win.X
        K = np.concatenate([Kw[:len(Kw) - X], Kt, Kw[len(Kw) - X:], K_x])
        V = np.concatenate([Vw[:len(Vw) - X], Vt, Vw[len(Vw) - X:], V_x])
        n = K.shape[0]
        nx = Q_x.shape[0]
        return self._attend(Q_x, np.arange(n - nx, n), rows, K, V, np.arange(n))
    _expect_caught(monkeypatch, (StreamOracle, "verify"), bad, TAIL_PINS)


def test_planted_tail_kept_across_steps(monkeypatch):
    """A tail that survives a window step is caught."""
    orig = ViewMajorWindow.step

    def bad(self, K_new, V_new):
        keep = (self.tail_K, self.tail_V)
        orig(self, K_new, V_new)
        self.tail_K, self.tail_V = keep
    _expect_caught(monkeypatch, (ViewMajorWindow, "step"), bad, TAIL_PINS)


# ------------------------------------------------ encoder attention (newest frame)

def _brute_frame(Q, K, V, views, n):
    """Scalar Python: each view's frame tokens attend to each other, nothing else."""
    nt, H, d = Q.shape
    Hkv = K.shape[1]
    G = H // Hkv
    out = np.zeros((nt, H, d))
    for v in range(views):
        for a in range(v * n, (v + 1) * n):
            for h in range(H):
                kv = h // G
                sc = [sum(float(Q[a, h, i]) * float(K[b, kv, i]) for i in range(d)) / math.sqrt(d)
                      for b in range(v * n, (v + 1) * n)]
                mx = max(sc)
                w = [math.exp(x - mx) for x in sc]
                tot = sum(w)
                for i in range(d):
                    out[a, h, i] = sum(w[j] * float(V[v * n + j, kv, i]) for j in range(n)) / tot
    return out


def pin_frame_brute(views=2, n=5, H=4, Hkv=2, d=8, seed=31):
    rng = np.random.default_rng(seed)
    Q = bf16_bits_to_f64(_rand(rng, views * n, H, d))
    K = bf16_bits_to_f64(_rand(rng, views * n, Hkv, d))
    V = bf16_bits_to_f64(_rand(rng, views * n, Hkv, d))
    np.testing.assert_allclose(so.frame_attention(Q, K, V, views, n), _brute_frame(Q, K, V, views, n),
                               rtol=0, atol=1e-12)


def pin_frame_is_sdpa_per_view(views=3, n=17, H=8, Hkv=2, d=16, seed=32):
    """Each view's frame is torch SDPA (float64, no mask, GQA) over that frame alone."""
    rng = np.random.default_rng(seed)
    Q = bf16_bits_to_f64(_rand(rng, views * n, H, d))
    K = bf16_bits_to_f64(_rand(rng, views * n, Hkv, d))
    V = bf16_bits_to_f64(_rand(rng, views * n, Hkv, d))
    got = so.frame_attention(Q, K, V, views, n)
    for v in range(views):
        r = slice(v * n, (v + 1) * n)
        q = torch.tensor(Q[r]).permute(1, 0, 2)[None]
        k = torch.tensor(K[r]).permute(1, 0, 2)[None]
        vv = torch.tensor(V[r]).permute(1, 0, 2)[None]
        o = torch.nn.functional.scaled_dot_product_attention(q, k, vv, is_causal=False, enable_gqa=True)
        np.testing.assert_allclose(got[r], o[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def pin_frame_permutation_and_isolation(views=2, n=9, H=2, Hkv=1, d=8, seed=33):
    """Bidirectional with no positions: permuting a frame's tokens permutes its
    output rows; changing one view's tokens leaves the other views' output alone."""
    rng = np.random.default_rng(seed)
    Q = bf16_bits_to_f64(_rand(rng, views * n, H, d))
    K = bf16_bits_to_f64(_rand(rng, views * n, Hkv, d))
    V = bf16_bits_to_f64(_rand(rng, views * n, Hkv, d))
    base = so.frame_attention(Q, K, V, views, n)
    perm = np.concatenate([rng.permutation(n) + v * n for v in range(views)])
    got = so.frame_attention(Q[perm], K[perm], V[perm], views, n)
    np.testing.assert_allclose(got, base[perm], rtol=0, atol=1e-12)
    K2, V2 = K.copy(), V.copy()
    K2[n:] = bf16_bits_to_f64(_rand(rng, (views - 1) * n, Hkv, d))
    V2[n:] = bf16_bits_to_f64(_rand(rng, (views - 1) * n, Hkv, d))
    np.testing.assert_array_equal(so.frame_attention(Q, K2, V2, views, n)[:n], base[:n])


FRAME_PINS = [pin_frame_brute, pin_frame_is_sdpa_per_view, pin_frame_permutation_and_isolation]


def test_frame_attention_pins():
    for pin in FRAME_PINS:
        pin()


def test_planted_frame_causal_mask(monkeypatch):
    """A causal mask inside the frame (the streaming path's habit) is caught."""
    def bad(Q, K, V, views, n):
        Q = np.asarray(Q, dtype=np.float64)
        out = np.empty(Q.shape)
        for v in range(views):
            r = slice(v * n, (v + 1) * n)
            pos = np.arange(n)
            out[r] = so.masked_attention(Q[r], pos, K[r], V[r], pos, 1.0)  # base 1.0: angle 0 only at pos 0
        return out
    _expect_caught(monkeypatch, (so, "frame_attention"), bad, FRAME_PINS)


def test_planted_frame_across_views(monkeypatch):
    """Attention that leaks across views is caught."""
    def bad(Q, K, V, views, n):
        return so.masked_attention(Q, np.zeros(len(Q)), K, V, np.zeros(len(K)), 10000.0)
    _expect_caught(monkeypatch, (so, "frame_attention"), bad, FRAME_PINS)


# ------------------------------------------------------------- K/V projection

def pin_bf16_round_definition(seed=41):
    """bf16_round returns a bf16 value (float32 with zero low 16 bits) at least as
    close as both neighbours, ties going to the even significand."""
    rng = np.random.default_rng(seed)
    x = np.concatenate([rng.standard_normal(2000) * np.exp2(rng.integers(-20, 20, 2000)),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 3.0, 0.0,
                                  1.0 + 2 ** -8 + 2 ** -30])])  # just above a tie: nearest is 1 + 2^-7
    b = so.bf16_round(x)
    b32 = b.astype(np.float32)
    assert np.array_equal(b32.astype(np.float64), b)
    assert not np.any(b32.view(np.uint32) & np.uint32(0xFFFF))
    for xi, bi in zip(x, b):
        if xi == 0:
            assert bi == 0
            continue
        bits = np.float32(bi).view(np.uint32)
        up = float(np.uint32(bits + np.uint32(0x10000)).view(np.float32))
        dn = float(np.uint32(bits - np.uint32(0x10000)).view(np.float32))
        err = abs(xi - bi)
        assert err <= abs(xi - up) and err <= abs(xi - dn), (xi, bi)
        if err == abs(xi - up) or err == abs(xi - dn):  # a tie: the even significand wins
            assert (bits >> np.uint32(16)) & np.uint32(1) == 0, (xi, bi)
    np.testing.assert_array_equal(so.bf16_round(np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8])), [1.0, 1.0 + 2 ** -6])


def pin_project_kv_brute(n=3, dm=6, Hkv=2, d=4, seed=42):
    rng = np.random.default_rng(seed)
    X = bf16_bits_to_f64(_rand(rng, n, dm))
    W = bf16_bits_to_f64(_rand(rng, 2 * Hkv * d, dm))
    K, V = so.project_kv(X, W, Hkv, d)
    for t in range(n):
        for o in range(2 * Hkv * d):
            y = 0.0
            for i in range(dm):
                y += float(X[t, i]) * float(W[o, i])
            want = so.bf16_round(np.array([y]))[0]
            got = K[t, o // d, o % d] if o < Hkv * d else V[t, (o - Hkv * d) // d, o % d]
            assert got == want, (t, o, got, want)


def test_projection_pins():
    pin_bf16_round_definition()
    pin_project_kv_brute()
    pin_project_kv_brute(n=5, dm=16, Hkv=1, d=8, seed=43)


def test_planted_projection_transposed(monkeypatch):
    """Using W's transpose layout (K from columns instead of rows) is caught."""
    def bad(X, W, Hkv, d):
        Y = so.bf16_round(np.asarray(X) @ np.asarray(W).reshape(np.asarray(W).shape[1], -1))
        n = Y.shape[0]
        return Y[:, :Hkv * d].reshape(n, Hkv, d), Y[:, Hkv * d:].reshape(n, Hkv, d)
    _expect_caught(monkeypatch, (so, "project_kv"), bad, [pin_project_kv_brute])


def test_planted_projection_double_rounding(monkeypatch):
    """Rounding through float32 first (double rounding) is caught: 1 + 2^-8 + 2^-30
    becomes the tie 1 + 2^-8 in float32 and then rounds to even (1.0), not to the
    nearest bf16 value 1 + 2^-7."""
    _expect_caught(monkeypatch, (so, "bf16_round"),
                   lambda x: torch.tensor(np.asarray(x, dtype=np.float64)).float().bfloat16().double().numpy(),
                   [pin_bf16_round_definition])
