"""Drive the CUDA library step by step and compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np

import oracle
import synth

OUT_TOL = 2e-3  # max-abs on out (fp32 path vs fp64 oracle)
LSE_TOL = 1e-3  # max-abs on lse


def torch_dev():
    import torch
    assert torch.cuda.is_available(), "GPU test without a CUDA device"
    return torch, torch.device("cuda:0")


class DeviceRun:
    """One MacState plus device copies of a workload's cache."""

    def __init__(self, wl, cache, tau=None, band=None, window=None, K_dev=None, V_dev=None, tune=None, cut_mode=0,
                 per_head=0, q_bf16=0, ring_bf16=0):
        import kv_cache_reuse_b200 as mac
        torch, dev = torch_dev()
        self.torch, self.dev, self.wl, self.cache = torch, dev, wl, cache
        self.K = K_dev if K_dev is not None else torch.from_numpy(cache.K.view(np.int16)).to(dev)
        self.V = V_dev if V_dev is not None else torch.from_numpy(cache.V.view(np.int16)).to(dev)
        self.bt = None if not cache.paged else torch.from_numpy(cache.block_table).to(dev)
        if cache.paged:
            self.st = mac.MacState.for_workload(wl, max_pages_per_seq=cache.block_table.shape[1],
                                                num_pages=cache.num_pages, tau=tau, band=band, window=window,
                                                cut_mode=cut_mode, match_per_head=per_head, q_bf16=q_bf16,
                                                ring_bf16=ring_bf16)
        else:
            self.st = mac.MacState.for_workload(wl, capacity=cache.max_seq, tau=tau, band=band, window=window,
                                                cut_mode=cut_mode, match_per_head=per_head, q_bf16=q_bf16,
                                                ring_bf16=ring_bf16)
        for name, val in (tune or {}).items():  # work-split knobs: min_keys_per_cta, piece_cost, whole_unit_keys
            getattr(mac, "mac_set_" + name)(self.st, val)
        B, Hq, Hkv, D = wl.B, wl.Hq, wl.Hkv, wl.D
        f32, i32 = torch.float32, torch.int32
        self.q_bf16 = q_bf16
        self.q = torch.empty((B, Hq, D), dtype=torch.int16 if q_bf16 else f32, device=dev)
        self.pos = torch.empty(B, dtype=i32, device=dev)
        self.lens = torch.empty(B, dtype=i32, device=dev)
        self.out = torch.empty((B, Hq, D), dtype=f32, device=dev)
        self.lse = torch.empty((B, Hq), dtype=f32, device=dev)
        nd = Hq if per_head else Hkv  # match decisions per sequence
        self.hit = torch.empty((B, nd), dtype=torch.uint8, device=dev)
        self.mpos = torch.empty((B, nd), dtype=i32, device=dev)

    def step(self, q, rope_pos, seq_lens):
        torch = self.torch
        if self.q_bf16:  # the bf16 bits of the query (the caller passes bf16-exact values)
            self.q.copy_(torch.from_numpy(synth.f32_to_bf16_bits(q).view(np.int16)))
        else:
            self.q.copy_(torch.from_numpy(np.ascontiguousarray(q, np.float32)))
        self.pos.copy_(torch.from_numpy(np.ascontiguousarray(rope_pos, np.int32)))
        self.lens.copy_(torch.from_numpy(np.ascontiguousarray(seq_lens, np.int32)))
        self.st.decode_step(self.q, self.pos, self.K, self.V, self.bt, self.lens, self.out, self.lse, self.hit,
                            self.mpos)
        torch.cuda.synchronize()
        return (self.out.cpu().numpy(), self.lse.cpu().numpy(), self.hit.cpu().numpy(), self.mpos.cpu().numpy())


def compare_stream(wl, stream, cache, steps=None, tau=None, band=None, window=None, gpu=None, orc=None,
                   rope_zero=False, tune=None, cut_mode=0, start=0, per_head=0, q_bf16=0, ring_bf16=0):
    """Run both sides over the stream; assert parity at every step.  Returns stats.
    With q_bf16 the queries are rounded to bf16 first: the library reads the
    bits, the oracle their exact values."""
    T = stream.q.shape[0] if steps is None else steps
    gpu = gpu or DeviceRun(wl, cache, tau=tau, band=band, window=window, tune=tune, cut_mode=cut_mode,
                        per_head=per_head, q_bf16=q_bf16, ring_bf16=ring_bf16)
    orc = orc or oracle.Oracle.for_workload(wl, cache, tau=tau, band=band, W=window, cut_mode=cut_mode,
                                            per_head=per_head, ring_bf16=ring_bf16)
    if q_bf16:
        stream = synth.QueryStream(q=synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(stream.q)), label=stream.label,
                                   src=stream.src, rope_pos=stream.rope_pos, seq_lens=stream.seq_lens)
    worst_o = worst_l = 0.0
    hits = 0
    for t in range(start, T):
        rp = np.zeros_like(stream.rope_pos[t]) if rope_zero else stream.rope_pos[t]
        r = orc.step(stream.q[t], rp, cache.K, cache.V, cache.block_table, stream.seq_lens[t])
        out, lse, hit, mpos = gpu.step(stream.q[t], rp, stream.seq_lens[t])
        np.testing.assert_array_equal(hit, r.hit, err_msg="hit mask, step %d" % t)
        np.testing.assert_array_equal(mpos, r.match_pos, err_msg="match position, step %d" % t)
        eo = float(np.abs(out - r.out).max())
        el = float(np.abs(lse - r.lse).max())
        assert eo <= OUT_TOL, "out max-abs %.3g at step %d" % (eo, t)
        assert el <= LSE_TOL, "lse max-abs %.3g at step %d" % (el, t)
        worst_o, worst_l = max(worst_o, eo), max(worst_l, el)
        hits += int(hit.sum())
    assert gpu.st.get_status() == 0
    return {"worst_out": worst_o, "worst_lse": worst_l, "hits": hits, "gpu": gpu, "oracle": orc}
