"""The allocation-free entry point (mac_dense_decode_static) against the
existing one.

Some callers of this library cannot allocate device memory: plugins inside
inference servers that must draw every byte from the host framework's
pre-planned pool, and latency-critical paths that cannot take an
allocation's implicit synchronisation.  mac_dense_decode_static serves them by
keeping its scratch in a static device array.  Here it must agree with the
regular entry point run with threshold 0 (every step a miss, i.e. dense
decode attention over all keys), on two calls in a row, because the second
call finds the scratch as the first left it.  This file is collected last so
that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest

import synth
from tests.gpu_harness import LSE_TOL, OUT_TOL, DeviceRun


def test_rejects_shapes_beyond_the_static_scratch():
    import kv_cache_reuse_b200 as mac
    mac.load()
    # 17 sequences x 4 KV heads = 68 units > 64: refused before any CUDA call
    rc = mac.mac_dense_decode_static(16, 16, 16, 16, None, 16, 16, 16, None, 17, 16, 4, 128, 5e5,
                                     0, 1024, 0, 0, 0)
    assert rc == mac.MAC_ERR_SHAPE
    # 4 sequences x 72 query heads = 288 query rows > 256
    rc = mac.mac_dense_decode_static(16, 16, 16, 16, None, 16, 16, 16, None, 4, 72, 9, 128, 5e5,
                                     0, 1024, 0, 0, 0)
    assert rc == mac.MAC_ERR_SHAPE
    # 9 query heads per KV head
    rc = mac.mac_dense_decode_static(16, 16, 16, 16, None, 16, 16, 16, None, 1, 18, 2, 128, 5e5,
                                     0, 1024, 0, 0, 0)
    assert rc == mac.MAC_ERR_SHAPE


@pytest.mark.gpu
@pytest.mark.parametrize("paged,Hq", [(False, 32), (True, 32), (False, 8), (True, 64)])
def test_static_scratch_matches_regular_entry_on_two_calls(paged, Hq):
    """Groups of 4, 1 (8 query heads over 8 KV heads) and 8 (64 over 8)."""
    import kv_cache_reuse_b200 as mac
    base = synth.WORKLOADS["paged_mixed" if paged else "llama8b_32k"]
    wl = base.with_(B=3, L0=(5000, 3210, 777), steps=2, Hq=Hq)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    ref = DeviceRun(wl, cache, tau=0.0)  # regular entry point, never hits: dense attention
    torch = ref.torch
    out = torch.empty_like(ref.out)
    lse = torch.empty_like(ref.lse)
    status = torch.zeros(1, dtype=torch.int32, device=ref.dev)
    bt = ref.bt
    for t in range(2):
        o_ref, l_ref, _, _ = ref.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        out.fill_(float("nan"))
        rc = mac.mac_dense_decode_static(
            ref.q, ref.pos, ref.K, ref.V, bt, ref.lens, out, lse, status, wl.B, wl.Hq, wl.Hkv, wl.D, wl.rope_theta,
            wl.page_size, 0 if paged else cache.max_seq, cache.block_table.shape[1] if paged else 0,
            cache.num_pages if paged else 0)
        assert rc == mac.MAC_OK
        torch.cuda.synchronize()
        o = out.cpu().numpy()
        l_ = lse.cpu().numpy()
        assert np.isfinite(o).all()
        assert float(np.abs(o - o_ref).max()) <= OUT_TOL
        assert float(np.abs(l_ - l_ref).max()) <= LSE_TOL
    assert int(status.item()) == 0
