"""MAC-Attention decode step on B200: Python binding of libmac_b200.so.

Argument marshalling only -- every stage of the step (match, RoPE, amend,
complete, miss fallback, merge, ring update) runs in the library's CUDA
kernels.  Tensors are torch tensors on the state's device (PyTorch is used for
device memory and streams); the functions carry the names of the C ABI in
include/mac.h and forward to it.  There is no CPU fallback: if the library is
missing, importing the native module raises.
"""
from __future__ import annotations

import ctypes as C
from typing import Optional

from ._native import (MAC_DEV_BAD_PAGE, MAC_DEV_BAD_SEQ_LEN, MAC_DEV_TIMEOUT, MAC_ERR_ARG, MAC_ERR_CUDA,
                      MAC_ERR_DEVICE, MAC_ERR_OOM, MAC_ERR_SHAPE, MAC_OK, LIB_PATH, MacConfig, MacError, check,
                      load)

__all__ = [
    "MacConfig", "MacError", "MacState", "mac_init_state", "mac_destroy", "mac_reset_seq", "mac_decode_step",
    "mac_match", "mac_attend", "mac_append_kv", "mac_decode_step_host", "mac_get_status", "mac_state_bytes",
    "mac_export_state", "mac_import_state", "mac_set_min_keys_per_cta", "mac_set_piece_cost", "mac_set_whole_unit_keys", "mac_warm_start", "mac_attend_grid", "mac_error_string", "mac_dense_decode_static",
    "mac_selftest_wait_timeout",
    "MAC_OK", "MAC_ERR_ARG", "MAC_ERR_SHAPE", "MAC_ERR_CUDA", "MAC_ERR_OOM", "MAC_ERR_DEVICE",
    "MAC_DEV_BAD_SEQ_LEN", "MAC_DEV_BAD_PAGE", "MAC_DEV_TIMEOUT", "LIB_PATH",
]


def _ptr(t) -> Optional[int]:
    """Device (or host) address of a tensor / numpy array / int, None for None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        if not t.is_contiguous():
            raise ValueError("tensor arguments must be contiguous")
        return t.data_ptr()
    if hasattr(t, "ctypes"):
        return t.ctypes.data
    raise TypeError("unsupported argument type %r" % type(t))


class _Kinds(dict):
    """Accepted element types, named by suffix ("float32" matches torch.float32
    and numpy float32); each dtype object seen is decided once and remembered."""

    def __init__(self, *names):
        super().__init__()
        self.names = names

    def __missing__(self, dtype):
        ok = self[dtype] = any(str(dtype).endswith(k) for k in self.names)
        return ok


_F32, _I32, _U8 = _Kinds("float32"), _Kinds("int32"), _Kinds("uint8", "bool")
_BF16 = _Kinds("int16", "uint16", "bfloat16")  # bf16 bit patterns


_tensor_cls = None  # torch.Tensor, once one has been seen (keeps torch a lazy import)


def _arg(t, name, shape, kinds, where=None):
    """Address of a tensor or array argument after checking it against the
    state's configuration: shape (or element count when shape is an int),
    element type, device ("cuda" or "cpu") and contiguity -- a mismatch would
    make the kernels read or write outside the caller's buffer.  None stays
    None; a raw integer address passes unchecked (the caller vouches for it)."""
    global _tensor_cls
    if t is None:
        return None
    c = t.__class__
    if c is int:
        return t
    if not kinds[t.dtype]:
        raise ValueError("%s: element type %s, expected one of %s" % (name, t.dtype, "/".join(kinds.names)))
    if shape.__class__ is int:
        n = t.numel() if hasattr(t, "numel") else t.size
        if n < shape:
            raise ValueError("%s: %d elements, the configuration needs %d" % (name, n, shape))
    elif t.shape != shape:
        raise ValueError("%s: shape %s, expected %s" % (name, tuple(t.shape), shape))
    if c is _tensor_cls or hasattr(t, "data_ptr"):
        _tensor_cls = c
        if where is not None and t.is_cuda != (where == "cuda"):
            raise ValueError("%s: expected a %s buffer" % (name, "device" if where == "cuda" else "host"))
        if not t.is_contiguous():
            raise ValueError("%s: tensor arguments must be contiguous" % name)
        return t.data_ptr()
    if where == "cuda":
        raise ValueError("%s: expected a device buffer" % name)
    if not t.flags.c_contiguous:
        raise ValueError("%s: arrays must be C-contiguous" % name)
    return t.ctypes.data


def _spec(st):
    """Expected shapes and element types of a state's buffers (computed once)."""
    sp = st.__dict__.get("_spec_cache")
    if sp is None:
        c = st.cfg
        B, Hq, Hkv, D = c.batch, c.num_q_heads, c.num_kv_heads, c.head_dim
        nd = Hq if c.match_per_head else Hkv
        rows = c.max_seq * B if c.page_size == 0 else c.num_pages * c.page_size
        sp = dict(B=B, Hq=Hq, Hkv=Hkv, D=D, q=(B, Hq, D), qk=_BF16 if c.q_bf16 else _F32, b=(B,), o=(B, Hq, D),
                  l=(B, Hq), d=(B, nd), kv=rows * Hkv * D, paged=c.page_size > 0, bt=(B, c.max_pages_per_seq),
                  row=(B, Hkv, D))
        st.__dict__["_spec_cache"] = sp
    return sp


def _args(st, where, q_pre=None, rope_pos=None, seq_lens=None, out=None, lse=None, hit=None, mpos=None, K=None,
          V=None, block_table=None, k_new=None, v_new=None, n=None):
    """Addresses of a step's arguments, in this order: q_pre, rope_pos,
    seq_lens, out, lse, hit_mask, match_pos, K, V, block_table, k_new, v_new.
    With a MacState each is checked against its configuration (the step's
    own buffers on `where`, the cache always on the device; n: leading
    dimension of q_pre, rope_pos and seq_lens for a warm start); a raw
    handle gets the addresses unchecked."""
    if not isinstance(st, MacState):
        return (_ptr(q_pre), _ptr(rope_pos), _ptr(seq_lens), _ptr(out), _ptr(lse), _ptr(hit), _ptr(mpos), _ptr(K),
                _ptr(V), _ptr(block_table), _ptr(k_new), _ptr(v_new))
    sp = _spec(st)
    q, b = (sp["q"], sp["b"]) if n is None else ((n,) + sp["q"], (n,) + sp["b"])
    return (_arg(q_pre, "q_pre", q, sp["qk"], where),
            _arg(rope_pos, "rope_pos", b, _I32, where),
            _arg(seq_lens, "seq_lens", b, _I32, where),
            _arg(out, "out", sp["o"], _F32, where),
            _arg(lse, "lse", sp["l"], _F32, where),
            _arg(hit, "hit_mask", sp["d"], _U8, where),
            _arg(mpos, "match_pos", sp["d"], _I32, where),
            _arg(K, "K", sp["kv"], _BF16, "cuda"),
            _arg(V, "V", sp["kv"], _BF16, "cuda"),
            _arg(block_table, "block_table", sp["bt"], _I32, "cuda") if sp["paged"] else _ptr(block_table),
            _arg(k_new, "k_new", sp["row"], _BF16, where),
            _arg(v_new, "v_new", sp["row"], _BF16, where))


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class MacState:
    """Owns one C MacState (ring buffers + scratch of one attention layer)."""

    def __init__(self, batch, num_q_heads, num_kv_heads, head_dim, window, band, tau, rope_theta,
                 page_size=0, max_seq=0, max_pages_per_seq=0, num_pages=0, cut_mode=0, match_per_head=0,
                 q_bf16=0, ring_bf16=0):
        self.cfg = MacConfig(batch, num_q_heads, num_kv_heads, head_dim, window, band, float(tau),
                             float(rope_theta), page_size, max_seq, max_pages_per_seq, num_pages, cut_mode,
                             match_per_head, q_bf16, ring_bf16)
        self.lib = load()
        h = C.c_void_p()
        check("mac_init_state", self.lib.mac_init_state(C.byref(self.cfg), C.byref(h)))
        self.handle = h

    @classmethod
    def for_workload(cls, wl, capacity=None, max_pages_per_seq=0, num_pages=0, tau=None, band=None, window=None,
                     cut_mode=0, match_per_head=0, q_bf16=0, ring_bf16=0):
        """State sized for a synth.Workload (contiguous capacity or paged pool)."""
        return cls(wl.B, wl.Hq, wl.Hkv, wl.D, wl.W if window is None else window,
                   wl.band if band is None else band, wl.tau if tau is None else tau, wl.rope_theta,
                   wl.page_size, capacity or 0, max_pages_per_seq, num_pages, cut_mode, match_per_head, q_bf16,
                   ring_bf16)

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            self.lib.mac_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # --- thin forwards -------------------------------------------------
    def decode_step(self, q_pre, rope_pos, K, V, block_table, seq_lens, out, lse, hit_mask=None, match_pos=None,
                    stream=None):
        return mac_decode_step(self, q_pre, rope_pos, K, V, block_table, seq_lens, out, lse, hit_mask, match_pos,
                               stream)

    def match(self, q_pre, rope_pos, block_table, seq_lens, out, lse, hit_mask=None, match_pos=None, stream=None):
        return mac_match(self, q_pre, rope_pos, block_table, seq_lens, out, lse, hit_mask, match_pos, stream)

    def attend(self, K, V, block_table, out, lse, stream=None):
        return mac_attend(self, K, V, block_table, out, lse, stream)

    def append_kv(self, K, V, block_table, seq_lens, k_new, v_new, stream=None):
        return mac_append_kv(self, K, V, block_table, seq_lens, k_new, v_new, stream)

    def reset_seq(self, b, stream=None):
        return mac_reset_seq(self, b, stream)

    def get_status(self) -> int:
        return mac_get_status(self)

    def export_state(self):
        return mac_export_state(self)

    def import_state(self, buf):
        return mac_import_state(self, buf)


def mac_init_state(cfg: MacConfig) -> C.c_void_p:
    h = C.c_void_p()
    check("mac_init_state", load().mac_init_state(C.byref(cfg), C.byref(h)))
    return h


def _h(st):
    return st.handle if isinstance(st, MacState) else st


def mac_destroy(st) -> None:
    if isinstance(st, MacState):
        st.close()
    else:
        load().mac_destroy(st)


def mac_reset_seq(st, b: int, stream=None) -> None:
    check("mac_reset_seq", load().mac_reset_seq(_h(st), int(b), _stream(stream)))


def mac_decode_step(st, q_pre, rope_pos, K, V, block_table, seq_lens, out, lse, hit_mask=None, match_pos=None,
                    stream=None) -> None:
    q, pz, ln, o, l, hm, mp, k, v, bt, _, _ = _args(st, "cuda", q_pre, rope_pos, seq_lens, out, lse, hit_mask,
                                                   match_pos, K, V, block_table)
    check("mac_decode_step", load().mac_decode_step(_h(st), q, pz, k, v, bt, ln, o, l, hm, mp, _stream(stream)))


def mac_match(st, q_pre, rope_pos, block_table, seq_lens, out, lse, hit_mask=None, match_pos=None,
              stream=None) -> None:
    q, pz, ln, o, l, hm, mp, _, _, bt, _, _ = _args(st, "cuda", q_pre, rope_pos, seq_lens, out, lse, hit_mask,
                                                   match_pos, block_table=block_table)
    check("mac_match", load().mac_match(_h(st), q, pz, bt, ln, o, l, hm, mp, _stream(stream)))


def mac_attend(st, K, V, block_table, out, lse, stream=None) -> None:
    _, _, _, o, l, _, _, k, v, bt, _, _ = _args(st, "cuda", out=out, lse=lse, K=K, V=V, block_table=block_table)
    check("mac_attend", load().mac_attend(_h(st), k, v, bt, o, l, _stream(stream)))


def mac_append_kv(st, K, V, block_table, seq_lens, k_new, v_new, stream=None) -> None:
    _, _, ln, _, _, _, _, k, v, bt, kn, vn = _args(st, "cuda", seq_lens=seq_lens, K=K, V=V, block_table=block_table,
                                                  k_new=k_new, v_new=v_new)
    check("mac_append_kv", load().mac_append_kv(_h(st), k, v, bt, ln, kn, vn, _stream(stream)))


def mac_decode_step_host(st, q_pre_h, rope_pos_h, seq_lens_h, k_new_h, v_new_h, K, V, block_table, out_h, lse_h,
                         hit_h=None, match_pos_h=None, stream=None) -> int:
    """Host-buffer step; returns MAC_OK or MAC_ERR_DEVICE (status word set)."""
    q, pz, ln, o, l, hm, mp, k, v, bt, kn, vn = _args(st, "cpu", q_pre_h, rope_pos_h, seq_lens_h, out_h, lse_h, hit_h,
                                                     match_pos_h, K, V, block_table, k_new_h, v_new_h)
    rc = load().mac_decode_step_host(_h(st), q, pz, ln, kn, vn, k, v, bt, o, l, hm, mp, _stream(stream))
    if rc not in (MAC_OK, MAC_ERR_DEVICE):
        check("mac_decode_step_host", rc)
    return rc


def mac_get_status(st) -> int:
    v = C.c_int(0)
    rc = load().mac_get_status(_h(st), C.byref(v))
    if rc not in (MAC_OK, MAC_ERR_DEVICE):
        check("mac_get_status", rc)
    return v.value


def mac_state_bytes(st) -> int:
    return int(load().mac_state_bytes(_h(st)))


def mac_export_state(st):
    import numpy as np
    buf = np.empty(mac_state_bytes(st), np.uint8)
    check("mac_export_state", load().mac_export_state(_h(st), buf.ctypes.data, buf.nbytes))
    return buf


def mac_import_state(st, buf) -> None:
    import numpy as np
    buf = np.ascontiguousarray(buf, np.uint8)
    check("mac_import_state", load().mac_import_state(_h(st), buf.ctypes.data, buf.nbytes))


def mac_set_min_keys_per_cta(st, keys: int) -> None:
    check("mac_set_min_keys_per_cta", load().mac_set_min_keys_per_cta(_h(st), int(keys)))


def mac_set_piece_cost(st, keys: int) -> None:
    check("mac_set_piece_cost", load().mac_set_piece_cost(_h(st), int(keys)))


def mac_warm_start(st, n: int, q_pre, rope_pos, K, V, block_table, seq_lens, stream=None) -> None:
    if n > 0:
        q, pz, ln, _, _, _, _, k, v, bt, _, _ = _args(st, "cuda", q_pre, rope_pos, seq_lens, K=K, V=V,
                                                     block_table=block_table, n=n)
    else:
        q, pz, ln, k, v, bt = _ptr(q_pre), _ptr(rope_pos), _ptr(seq_lens), _ptr(K), _ptr(V), _ptr(block_table)
    check("mac_warm_start", load().mac_warm_start(_h(st), int(n), q, pz, k, v, bt, ln, _stream(stream)))


def mac_set_whole_unit_keys(st, keys: int) -> None:
    check("mac_set_whole_unit_keys", load().mac_set_whole_unit_keys(_h(st), int(keys)))


def mac_set_reproducible(st, on: int) -> None:
    check("mac_set_reproducible", load().mac_set_reproducible(_h(st), int(on)))


def mac_set_one_launch(st, on: int) -> None:
    check("mac_set_one_launch", load().mac_set_one_launch(_h(st), int(on)))


def mac_one_launch(st) -> int:
    return int(load().mac_one_launch(_h(st)))


def mac_set_trace(st, on: int) -> None:
    check("mac_set_trace", load().mac_set_trace(_h(st), int(on)))


def mac_get_trace(st):
    """(stamps [grid][12] uint64 ns of the last traced step's phases, counters [4]
    uint64 since the last call: keys attended fresh, pieces, whole units, merges)."""
    import numpy as np
    g = mac_attend_grid(st)
    stamps = np.zeros((g, 12), np.uint64)
    counters = np.zeros(4, np.uint64)
    check("mac_get_trace", load().mac_get_trace(_h(st), stamps.ctypes.data, stamps.size, counters.ctypes.data))
    return stamps, counters


def mac_attend_grid(st) -> int:
    return int(load().mac_attend_grid(_h(st)))


def mac_dense_decode_static(q_pre, rope_pos, K, V, block_table, seq_lens, out, lse, device_status, batch,
                            num_q_heads, num_kv_heads, head_dim, rope_theta, page_size=0, max_seq=0,
                            max_pages_per_seq=0, num_pages=0, stream=None) -> int:
    """Dense decode attention whose scratch is the library's static device
    array (no allocation); returns the C return code."""
    return int(load().mac_dense_decode_static(
        _ptr(q_pre), _ptr(rope_pos), _ptr(K), _ptr(V), _ptr(block_table), _ptr(seq_lens), _ptr(out), _ptr(lse),
        _ptr(device_status), int(batch), int(num_q_heads), int(num_kv_heads), int(head_dim), float(rope_theta),
        int(page_size), int(max_seq), int(max_pages_per_seq), int(num_pages), _stream(stream)))


def mac_selftest_wait_timeout(device_status, stream=None) -> None:
    """Enqueue the failure-path self-test: a kernel whose bounded wait runs out
    (about 2 s) and ORs MAC_DEV_TIMEOUT into device_status."""
    check("mac_selftest_wait_timeout", load().mac_selftest_wait_timeout(_ptr(device_status), _stream(stream)))


def mac_error_string(code: int) -> str:
    return load().mac_error_string(int(code)).decode()


def parse_state(buf, W: int, G: int, D: int):
    """Split an exported state buffer into named numpy arrays (layout of include/mac.h);
    a bf16 window's q and o come back as their bf16 bit patterns (uint16)."""
    import numpy as np
    hdr = np.frombuffer(buf[:32].tobytes(), np.int32)
    U, W1 = int(hdr[1]), int(hdr[2])
    qt = np.uint16 if int(hdr[5]) else np.float32
    off = 32
    out = {}
    for name, n, dt, shape in (("q", U * W1 * G * D, qt, (U, W1, G, D)),
                               ("o", U * W1 * G * D, qt, (U, W1, G, D)),
                               ("m", U * W1 * G, np.float32, (U, W1, G)),
                               ("l", U * W1 * G, np.float32, (U, W1, G)),
                               ("pos", U * W1, np.int32, (U, W1)),
                               ("steps", U, np.int32, (U,))):
        nb = n * np.dtype(dt).itemsize
        out[name] = np.frombuffer(buf[off:off + nb].tobytes(), dt).reshape(shape)
        off += nb
    return out
