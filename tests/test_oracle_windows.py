"""Pins of the oracle's bf16 token windows.

Sources: Dual-QK summary Sec. 3.3 (the first 64 and the most recent 256
tokens remain BF16); tq-kv abstract (sink-token preservation).  Window tokens
are kept as bf16 copies of the rotated key and of the value (rotated when
values are) and scored over every channel; the other tokens come from the
codes (with the channel mask); one softmax covers both.  Token n < sink sits
in slot n, token n >= sink in ring slot sink + (n - sink) % recent; a decode of
a length-len sequence takes tokens n < sink and n >= max(sink, len - recent)
from the window.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as orc


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def draw(seed, H, T):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((1, H, T, 128)).astype(np.float32)
    v = (rng.standard_normal((1, H, T, 128)) * 0.8 + 0.1).astype(np.float32)
    q = rng.standard_normal((1, 2 * H, 128)).astype(np.float32)
    return q, k, v


def rot_rows(x):
    return np.stack([orc.rotate(r) for r in x.reshape(-1, 128)]).reshape(x.shape)


@pytest.mark.parametrize("sink,recent,rotv", [(4, 8, 0), (0, 16, 1), (16, 0, 0), (5, 7, 1)])
def test_window_slots_hold_bf16_rotated_rows(sink, recent, rotv):
    H, T, off = 2, 50, 3
    _, k, v = draw(1 + sink + recent, H, T)
    c = orc.Cache(1, H, 128, 128, 4, 2, 1, 0, rotv, 1.0, sink, recent)
    c.append(k[:, :, :20], v[:, :, :20], off)
    c.append(k[:, :, 20:], v[:, :, 20:], off + 20)
    kw = c.k_win.reshape(H, sink + recent, 128)
    vw = c.v_win.reshape(H, sink + recent, 128)
    want_k = np.zeros((H, sink + recent, 128))
    want_v = np.zeros((H, sink + recent, 128))
    kr = rot_rows(k[0])
    vr = rot_rows(v[0]) if rotv else v[0].astype(np.float64)
    for t in range(T):  # appends write in token order; a ring slot keeps its last token
        n = off + t
        slot = n if n < sink else (sink + (n - sink) % recent if recent else None)
        if slot is not None:
            want_k[:, slot] = bf16(kr[:, t])
            want_v[:, slot] = bf16(vr[:, t])
    got_k = np.vectorize(orc.bf16_value)(kw)
    got_v = np.vectorize(orc.bf16_value)(vw)
    np.testing.assert_array_equal(got_k, want_k)
    np.testing.assert_array_equal(got_v, want_v)


def test_all_window_tokens_is_exact_bf16_attention():
    # a sink as long as the sequence: no token comes from the codes
    H, T = 2, 40
    q, k, v = draw(7, H, T)
    c = orc.Cache(1, H, 128, 128, 2, 2, 1, 1, 0, 1.0, 64, 0)
    c.append(k, v, 0)
    out = c.attention(q, np.array([T], np.int32), None, 1.0 / np.sqrt(128))
    kb, vb = bf16(rot_rows(k[0])), bf16(v[0])
    for hq in range(2 * H):
        h = hq // 2
        qr = orc.rotate(q[0, hq]).astype(np.float64)
        s = kb[h] @ qr / np.sqrt(128)
        p = np.exp(s - s.max())
        np.testing.assert_allclose(out[hq], (p / p.sum()) @ vb[h], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("sink,recent,rotv", [(4, 8, 0), (3, 16, 1), (0, 12, 0), (6, 0, 0)])
def test_mixed_sequences_assemble_window_and_code_tokens(sink, recent, rotv):
    # the recent ring holds the last tokens appended, so each length gets its
    # own cache holding exactly that many tokens
    H, T = 2, 60
    q, k, v = draw(11 + recent, H, T)
    mask = np.array([[0x0F0F0F0F, 0xFFFFFFF0]], np.uint32)
    sel = [np.array([(int(mask[0, h]) >> (ch // 4)) & 1 for ch in range(128)], bool) for h in range(H)]
    kr = bf16(rot_rows(k[0]))
    vr = bf16(rot_rows(v[0]) if rotv else v[0])
    for L in (1, sink + 1, sink + recent - 1, 25, T):
        if L < 1 or L > T:
            continue
        c = orc.Cache(1, H, 128, 128, 4, 4, 1, 1, rotv, 0.92 if rotv else 1.0, sink, recent)
        c.append(k[:, :, :L], v[:, :, :L], 0)
        out = c.attention(q, np.array([L], np.int32), mask, 1.0 / np.sqrt(128))
        for hq in range(2 * H):
            h = hq // 2
            qr = orc.rotate(q[0, hq]).astype(np.float64)
            khat, vhat = c.dequantize(0, h, 0, L)
            s = np.empty(L)
            vv = np.empty((L, 128))
            for j in range(L):
                if j < sink or (recent and j >= max(sink, L - recent)):
                    s[j] = kr[h, j] @ qr
                    vv[j] = vr[h, j]
                else:
                    s[j] = khat[j, sel[h]] @ qr[sel[h]]
                    vv[j] = vhat[j]
            p = np.exp(s / np.sqrt(128) - (s / np.sqrt(128)).max())
            o = (p / p.sum()) @ vv
            if rotv:
                o = orc.fwht(o) / np.sqrt(128)
            np.testing.assert_allclose(out[hq], o, rtol=1e-10, atol=1e-12)


def test_windows_off_is_the_plain_cache():
    H, T = 2, 30
    q, k, v = draw(3, H, T)
    a = orc.Cache(1, H, 128, 128, 4, 2, 1, 1)
    b = orc.Cache(1, H, 128, 128, 4, 2, 1, 1, 0, 1.0, 0, 0)
    a.append(k, v, 0)
    b.append(k, v, 0)
    lens = np.array([T], np.int32)
    np.testing.assert_array_equal(a.attention(q, lens, None, 0.1), b.attention(q, lens, None, 0.1))
