"""Independent textbook references used to pin the oracle (numpy, fp64).

Nothing here is shared with the oracle's C code: RoPE is written as a complex
rotation, attention as a plain softmax over all scores.
"""
import json
import os

import numpy as np

from synth import bf16_bits_to_f32

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rope_complex(q: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """RoPE as multiplication of z_i = q_i + j q_{i+D/2} by exp(j pos theta^(-2i/D))."""
    q = np.asarray(q, np.float64)
    D = q.shape[-1]
    half = D // 2
    freq = theta ** (-2.0 * np.arange(half) / D)
    z = (q[..., :half] + 1j * q[..., half:]) * np.exp(1j * pos * freq)
    return np.concatenate([z.real, z.imag], axis=-1)


def dense_attention(qrot: np.ndarray, K: np.ndarray, V: np.ndarray):
    """softmax(qrot K^T / sqrt(D)) V and its natural-log log-sum-exp.

    qrot [H, D] fp64; K, V [L, D] fp64 (already decoded).  Returns (o [H, D], lse [H]).
    """
    D = qrot.shape[-1]
    s = qrot @ K.T / np.sqrt(D)
    mx = s.max(axis=-1, keepdims=True)
    w = np.exp(s - mx)
    den = w.sum(axis=-1, keepdims=True)
    return (w @ V) / den, (mx + np.log(den))[..., 0]


def decode(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)


def seq_kv(cache, b: int, kvh: int, L: int):
    """Decoded [L, D] K and V of sequence b, KV head kvh (contiguous or paged)."""
    if not cache.paged:
        return decode(cache.K[b, :L, kvh]), decode(cache.V[b, :L, kvh])
    ps = cache.K.shape[1]
    pages = cache.block_table[b, : (L + ps - 1) // ps]
    Kp = cache.K[pages][:, :, kvh].reshape(-1, cache.K.shape[-1])[:L]
    Vp = cache.V[pages][:, :, kvh].reshape(-1, cache.V.shape[-1])[:L]
    return decode(Kp), decode(Vp)


def dense_step(wl, cache, q_pre: np.ndarray, rope_pos, seq_lens):
    """Dense decode attention of every query head over all visible keys."""
    out = np.empty((wl.B, wl.Hq, wl.D))
    lse = np.empty((wl.B, wl.Hq))
    G = wl.Hq // wl.Hkv
    for b in range(wl.B):
        for kvh in range(wl.Hkv):
            K, V = seq_kv(cache, b, kvh, int(seq_lens[b]))
            qr = np.stack([rope_complex(q_pre[b, kvh * G + h], int(rope_pos[b]), wl.rope_theta) for h in range(G)])
            o, l = dense_attention(qr, K, V)
            out[b, kvh * G:(kvh + 1) * G] = o
            lse[b, kvh * G:(kvh + 1) * G] = l
    return out, lse


def load_hand_example():
    with open(os.path.join(GOLDEN, "hand_hit_example.json")) as f:
        g = json.load(f)
    sh = g["shape"]
    L, D = sh["max_seq"], sh["D"]
    Kf = np.zeros((1, L, 1, D), np.float32)
    Vf = np.zeros((1, L, 1, D), np.float32)
    Kf[0, :, 0, 0] = [1, 0, 0, 0, 1]
    Vf[0, :, 0, 0] = np.arange(L)
    Vf[0, :, 0, 1] = 1
    from synth import f32_to_bf16_bits
    K = f32_to_bf16_bits(Kf)
    V = f32_to_bf16_bits(Vf)
    q0 = {"8*ln(2)": 8 * np.log(2.0), "8*ln(4)": 8 * np.log(4.0)}
    qs = []
    for st in g["steps"]:
        q = np.zeros((1, sh["Hq"], D), np.float32)
        q[0, :, 0] = np.float32(q0[st["q0"]])
        qs.append(q)
    return g, K, V, qs
