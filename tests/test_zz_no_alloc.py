"""The allocation-free entry point (mac_dense_decode_static) against the fp64
oracle.

Some callers of this library cannot allocate device memory: plugins inside
inference servers that must draw every byte from the host framework's
pre-planned pool, and latency-critical paths that cannot take an
allocation's implicit synchronisation.  mac_dense_decode_static serves them by
keeping its scratch in a static device array.  It computes dense decode
attention over all keys, which is what the oracle computes with threshold 0
(every step a miss); each case runs two calls in a row, because the second
call finds the scratch as the first left it.  This file is collected last so
that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_harness import LSE_TOL, OUT_TOL, torch_dev


def test_rejects_shapes_beyond_the_static_scratch():
    import kv_cache_reuse_b200 as mac
    mac.load()
    # 17 sequences x 4 KV heads = 68 units > 64: refused before any CUDA call
    rc = mac.mac_dense_decode_static(16, 16, 16, 16, None, 16, 16, 16, 16, 17, 16, 4, 128, 5e5,
                                     0, 1024, 0, 0, 0)
    assert rc == mac.MAC_ERR_SHAPE
    # 4 sequences x 72 query heads = 288 query rows > 256
    rc = mac.mac_dense_decode_static(16, 16, 16, 16, None, 16, 16, 16, 16, 4, 72, 9, 128, 5e5,
                                     0, 1024, 0, 0, 0)
    assert rc == mac.MAC_ERR_SHAPE
    # 9 query heads per KV head
    rc = mac.mac_dense_decode_static(16, 16, 16, 16, None, 16, 16, 16, 16, 1, 18, 2, 128, 5e5,
                                     0, 1024, 0, 0, 0)
    assert rc == mac.MAC_ERR_SHAPE


def test_requires_a_status_word():
    """Without a status word a bad length or page id could not reach the
    caller: a NULL one is refused on the host."""
    import kv_cache_reuse_b200 as mac
    mac.load()
    rc = mac.mac_dense_decode_static(16, 16, 16, 16, None, 16, 16, 16, None, 1, 32, 8, 128, 5e5,
                                     0, 1024, 0, 0, 0)
    assert rc == mac.MAC_ERR_ARG


class _StaticCall:
    """Device buffers for one workload and the static entry's arguments."""

    def __init__(self, wl, cache):
        torch, dev = torch_dev()
        self.torch, self.wl, self.cache = torch, wl, cache
        self.K = torch.from_numpy(cache.K.view(np.int16)).to(dev)
        self.V = torch.from_numpy(cache.V.view(np.int16)).to(dev)
        self.bt = torch.from_numpy(cache.block_table).to(dev) if cache.paged else None
        self.q = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.float32, device=dev)
        self.pos = torch.empty(wl.B, dtype=torch.int32, device=dev)
        self.lens = torch.empty(wl.B, dtype=torch.int32, device=dev)
        self.out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.float32, device=dev)
        self.lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def __call__(self, q, rope_pos, seq_lens):
        import kv_cache_reuse_b200 as mac
        torch, wl, c = self.torch, self.wl, self.cache
        self.q.copy_(torch.from_numpy(np.ascontiguousarray(q, np.float32)))
        self.pos.copy_(torch.from_numpy(np.ascontiguousarray(rope_pos, np.int32)))
        self.lens.copy_(torch.from_numpy(np.ascontiguousarray(seq_lens, np.int32)))
        self.out.fill_(float("nan"))
        self.lse.fill_(float("nan"))
        rc = mac.mac_dense_decode_static(
            self.q, self.pos, self.K, self.V, self.bt, self.lens, self.out, self.lse, self.status, wl.B, wl.Hq,
            wl.Hkv, wl.D, wl.rope_theta, wl.page_size, 0 if c.paged else c.max_seq,
            c.block_table.shape[1] if c.paged else 0, c.num_pages if c.paged else 0)
        assert rc == mac.MAC_OK
        torch.cuda.synchronize()
        return self.out.cpu().numpy(), self.lse.cpu().numpy()


def _against_oracle(wl, calls=2):
    """`calls` calls in a row of the static entry on the workload's first steps,
    each against the fp64 oracle with threshold 0 (dense attention)."""
    stream, cache = synth.queries(wl, calls), synth.kv_cache(wl, calls)
    run = _StaticCall(wl, cache)
    orc = oracle.Oracle.for_workload(wl, cache, tau=0.0)
    for t in range(calls):
        ref = orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, cache.block_table, stream.seq_lens[t])
        assert not ref.hit.any()
        o, l_ = run(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        assert np.isfinite(o).all() and np.isfinite(l_).all()
        eo, el = float(np.abs(o - ref.out).max()), float(np.abs(l_ - ref.lse).max())
        assert eo <= OUT_TOL, "out max-abs %.3g, call %d" % (eo, t)
        assert el <= LSE_TOL, "lse max-abs %.3g, call %d" % (el, t)
    assert int(run.status.item()) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("paged,Hq", [(False, 32), (True, 32), (False, 8), (True, 64)])
def test_static_scratch_matches_oracle_on_two_calls(paged, Hq):
    """Groups of 4, 1 (8 query heads over 8 KV heads) and 8 (64 over 8),
    contiguous and paged K/V."""
    base = synth.WORKLOADS["paged_mixed" if paged else "llama8b_32k"]
    _against_oracle(base.with_(B=3, L0=(5000, 3210, 777), steps=2, Hq=Hq))


@pytest.mark.gpu
def test_static_frequencies_follow_head_dim_and_theta():
    """The inverse RoPE frequencies kept in the static array are replaced when
    a call's head_dim or rope_theta differs from the previous call's: D = 128,
    then D = 64, then D = 128 with another theta, each against the oracle."""
    llama, tiny = synth.WORKLOADS["llama8b_32k"], synth.WORKLOADS["tiny"]
    for wl in (llama.with_(B=2, L0=(3000, 1200), steps=2),
               tiny.with_(B=2, L0=(2000, 900), steps=2),
               llama.with_(B=2, L0=(3000, 1200), steps=2, rope_theta=1e4)):
        _against_oracle(wl)
