"""The C ABI library builds for sm_100a, loads without a GPU and exports every
entry point include/mac.h declares; the binding refuses to run without it."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "mac.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mac_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from kv_cache_reuse_b200 import build
    build.build()
    import kv_cache_reuse_b200 as mac
    return mac.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n


def test_binding_declares_every_symbol():
    from kv_cache_reuse_b200._native import SIGNATURES
    assert sorted(SIGNATURES) == _declared()


def test_error_strings(lib):
    import kv_cache_reuse_b200 as mac
    assert mac.mac_error_string(mac.MAC_OK) == "ok"
    assert "status" in mac.mac_error_string(mac.MAC_ERR_DEVICE)


def test_missing_library_fails_loudly(tmp_path):
    from kv_cache_reuse_b200 import _native
    with pytest.raises(ImportError):
        _native._lib_backup = _native._lib
        try:
            _native._lib = None
            _native.load(str(tmp_path / "nope.so"))
        finally:
            _native._lib = _native._lib_backup



def test_tuning_setters_reject_bad_handles(lib):
    """Every setter validates its arguments on the host (NULL state -> MAC_ERR_ARG)."""
    import kv_cache_reuse_b200 as mac
    for name in ("mac_set_min_keys_per_cta", "mac_set_piece_cost", "mac_set_whole_unit_keys",
                 "mac_set_reproducible"):
        with pytest.raises(mac.MacError) as e:
            getattr(mac, name)(None, 4)
        assert e.value.code == mac.MAC_ERR_ARG


def test_init_rejects_bad_config_before_touching_the_device(lib):
    """Configuration checks run on the host first: a bad cut mode, band or shape
    is refused without a GPU."""
    import kv_cache_reuse_b200 as mac
    for kw, code in ((dict(cut_mode=2), mac.MAC_ERR_ARG), (dict(cut_mode=-1), mac.MAC_ERR_ARG),
                     (dict(match_per_head=2), mac.MAC_ERR_ARG),
                     (dict(band=-1), mac.MAC_ERR_ARG), (dict(num_q_heads=20), mac.MAC_ERR_SHAPE),
                     (dict(num_q_heads=72), mac.MAC_ERR_SHAPE),  # 9 query heads per KV head
                     (dict(num_q_heads=96), mac.MAC_ERR_SHAPE),  # 12: larger groups are 16, 32 or 64
                     (dict(num_q_heads=1024), mac.MAC_ERR_SHAPE),  # 128 per KV head
                     (dict(num_q_heads=128, match_per_head=1), mac.MAC_ERR_SHAPE),  # per-head: up to 8
                     (dict(head_dim=96), mac.MAC_ERR_SHAPE)):
        args = dict(batch=1, num_q_heads=32, num_kv_heads=8, head_dim=128, window=8, band=16, tau=0.1,
                    rope_theta=1e4, max_seq=64)
        args.update(kw)
        with pytest.raises(mac.MacError) as e:
            mac.MacState(**args)
        assert e.value.code == code, kw


def test_warm_start_rejects_bad_arguments(lib):
    import kv_cache_reuse_b200 as mac
    with pytest.raises(mac.MacError) as e:
        mac.mac_warm_start(None, 1, 16, 16, 16, 16, None, 16, stream=0)
    assert e.value.code == mac.MAC_ERR_ARG


def test_binding_rejects_buffers_that_do_not_fit_the_state(lib):
    """A tensor whose shape, element type or device does not match the state's
    configuration is refused in the binding, before anything reaches a kernel
    (the kernels would read or write outside it)."""
    import torch
    import kv_cache_reuse_b200 as mac
    st = mac.MacState.__new__(mac.MacState)  # configuration only, no device state
    st.cfg = mac.MacConfig(2, 8, 2, 64, 4, 8, 0.1, 1e4, 0, 100, 0, 0, 0, 0, 0, 0)
    st.handle = None
    B, Hq, Hkv, D = 2, 8, 2, 64
    ok = dict(q_pre=torch.zeros(B, Hq, D), rope_pos=torch.zeros(B, dtype=torch.int32),
              seq_lens=torch.zeros(B, dtype=torch.int32), out=torch.zeros(B, Hq, D), lse=torch.zeros(B, Hq))
    for name, bad in (("q_pre", torch.zeros(B, Hkv, D)), ("q_pre", torch.zeros(B, Hq, D, dtype=torch.float64)),
                      ("out", torch.zeros(B, Hq, D - 1)), ("lse", torch.zeros(B, Hq, dtype=torch.int32)),
                      ("seq_lens", torch.zeros(B + 1, dtype=torch.int32))):
        args = dict(ok, **{name: bad})
        with pytest.raises(ValueError):
            mac.mac_match(st, args["q_pre"], args["rope_pos"], None, args["seq_lens"], args["out"], args["lse"])
    # host buffers are refused where device buffers are expected
    with pytest.raises(ValueError, match="device"):
        mac.mac_match(st, ok["q_pre"], ok["rope_pos"], None, ok["seq_lens"], ok["out"], ok["lse"])
    # a cache smaller than the configured capacity
    with pytest.raises(ValueError, match="elements"):
        mac.mac_attend(st, torch.zeros(B * 99 * Hkv * D, dtype=torch.int16), 16, None, 16, 16)


def _state_of(**kw):
    """A MacState carrying only a configuration (no device state), for the binding's checks."""
    import kv_cache_reuse_b200 as mac
    f = dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=64, window=4, band=8, tau=0.1, rope_theta=1e4,
             page_size=0, max_seq=100, max_pages_per_seq=0, num_pages=0, cut_mode=0, match_per_head=0, q_bf16=0,
             ring_bf16=0)
    f.update(kw)
    st = mac.MacState.__new__(mac.MacState)
    st.cfg = mac.MacConfig(*[f[name] for name, _ in mac.MacConfig._fields_])
    st.handle = None
    return st


def test_binding_checks_follow_the_configuration(lib):
    """The expected shapes and element types follow the state: per-head
    matching reports a decision per query head, a bf16 query is bf16 bits, a
    paged cache needs its block table, a warm start has a leading position
    dimension; host arrays are accepted where host buffers are expected, raw
    integer addresses pass unchecked, non-contiguous tensors are refused."""
    import numpy as np
    import torch
    from kv_cache_reuse_b200 import _args
    B, Hq, Hkv, D = 2, 8, 2, 64
    q, p = torch.zeros(B, Hq, D), torch.zeros(B, dtype=torch.int32)
    o, l = torch.zeros(B, Hq, D), torch.zeros(B, Hq)
    # per-head matching: hit mask and match positions are [B][Hq]
    ph = _state_of(match_per_head=1)
    a = _args(ph, "cpu", q, p, p, o, l, torch.zeros(B, Hq, dtype=torch.uint8), torch.zeros(B, Hq, dtype=torch.int32))
    assert all(isinstance(x, int) for x in a[:7])
    with pytest.raises(ValueError, match="hit_mask"):
        _args(ph, "cpu", q, p, p, o, l, torch.zeros(B, Hkv, dtype=torch.uint8))
    # bf16 query input: bf16 bits (int16 / uint16 / bfloat16), not fp32
    qb = _state_of(q_bf16=1)
    for dt in (torch.int16, torch.bfloat16):
        assert _args(qb, "cpu", torch.zeros(B, Hq, D, dtype=dt))[0]
    with pytest.raises(ValueError, match="q_pre"):
        _args(qb, "cpu", q)
    # paged cache: the block table is [B][max_pages] int32 on the device
    pg = _state_of(page_size=16, max_seq=0, max_pages_per_seq=5, num_pages=20)
    with pytest.raises(ValueError, match="block_table: shape"):
        _args(pg, "cuda", block_table=torch.zeros(B, 4, dtype=torch.int32))
    with pytest.raises(ValueError, match="block_table: expected a device"):
        _args(pg, "cuda", block_table=torch.zeros(B, 5, dtype=torch.int32))
    with pytest.raises(ValueError, match="K: .*elements"):
        _args(pg, "cuda", K=torch.zeros(20 * 16 * Hkv * D - 1, dtype=torch.int16))
    # warm start: [n][B][Hq][D] queries, [n][B] positions and lengths
    st = _state_of()
    assert _args(st, "cpu", torch.zeros(3, B, Hq, D), torch.zeros(3, B, dtype=torch.int32), n=3)[0]
    with pytest.raises(ValueError, match="q_pre"):
        _args(st, "cpu", q, n=3)
    # host arrays, raw addresses, contiguity
    assert _args(st, "cpu", np.zeros((B, Hq, D), np.float32))[0]
    with pytest.raises(ValueError, match="element type"):
        _args(st, "cpu", np.zeros((B, Hq, D), np.float64))
    with pytest.raises(ValueError, match="device buffer"):
        _args(st, "cuda", np.zeros((B, Hq, D), np.float32))
    assert _args(st, "cuda", 12345)[0] == 12345
    with pytest.raises(ValueError, match="contiguous"):
        _args(st, "cpu", torch.zeros(B, D, Hq).transpose(1, 2))


def test_config_struct_layout_matches_the_header(tmp_path):
    """The binding's MacConfig has the C header's size and field offsets: a C
    program built here from include/mac.h prints them (gcc, no GPU)."""
    import ctypes
    import subprocess
    from kv_cache_reuse_b200._native import MacConfig
    names = [n for n, _ in MacConfig._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include "mac.h"\nint main(void) {\n  printf("%zu\\n", sizeof(MacConfig));\n'
                   + "".join('  printf("%%zu\\n", offsetof(MacConfig, %s));\n' % n for n in names) + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    vals = [int(x) for x in subprocess.check_output([str(exe)]).decode().split()]
    assert vals[0] == ctypes.sizeof(MacConfig)
    assert vals[1:] == [getattr(MacConfig, n).offset for n in names]


def test_every_entry_point_is_documented_in_the_header():
    """Each function include/mac.h declares comes with a comment (its own, or
    the one heading the group of declarations it belongs to)."""
    src = open(os.path.join(ROOT, "include", "mac.h")).read()
    code = re.sub(r"/\*.*?\*/", lambda m: "\0" * len(m.group(0)), src, flags=re.S)  # keep offsets
    decl = re.compile(r"^[A-Za-z_][\w \t\*]*\b(mac_[a-z_]+)\s*\(", re.M)
    documented = {}
    prev_end, prev_name = 0, None
    for m in decl.finditer(code):
        between = src[prev_end:m.start()]
        has_comment = "*/" in between
        blank_line = "\n\n" in between.replace("\0", "")
        if has_comment:
            documented[m.group(1)] = True
        elif prev_name is not None and not blank_line:
            documented[m.group(1)] = documented[prev_name]  # same group as the declaration above
        else:
            documented[m.group(1)] = False
        prev_end, prev_name = code.index(";", m.end()) + 1, m.group(1)
    assert len(documented) >= 15
    assert all(documented.values()), sorted(n for n, ok in documented.items() if not ok)
