"""CUDA path vs the fp64 oracle, through the C ABI (libmac_b200.so).

Bar (MAC-Attention, page 1, with this library's readings): hit/miss flags and
matched positions bit-exact; out within 2e-3 max-abs; lse within 1e-3.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.dense_ref import load_hand_example
from tests.gpu_harness import LSE_TOL, OUT_TOL, DeviceRun, compare_stream, torch_dev

pytestmark = pytest.mark.gpu


def test_hand_worked_example_on_gpu():
    g, K, V, qs = load_hand_example()
    sh = g["shape"]
    wl = synth.Workload(name="hand", B=1, Hq=sh["Hq"], Hkv=sh["Hkv"], D=sh["D"], L0=(3,), steps=2, W=sh["W"],
                        band=sh["band"], tau=sh["tau"], sigma=0.0, rope_theta=sh["rope_theta"], page_size=0,
                        hit_model=("iid", 0.0), seed=0)
    cache = synth.KVCache(K, V, None, sh["max_seq"], 0)
    gpu = DeviceRun(wl, cache)
    for st, q in zip(g["steps"], qs):
        out, lse, hit, mpos = gpu.step(q, np.array([st["rope_pos"]], np.int32), np.array([st["seq_len"]], np.int32))
        assert int(hit[0, 0]) == st["hit"] and int(mpos[0, 0]) == st["match_pos"]
        np.testing.assert_allclose(out[0, :, 0], st["out0"], atol=1e-5)
        np.testing.assert_allclose(out[0, :, 1], st["out1"], atol=1e-5)
        assert np.abs(out[0, :, 2:]).max() == 0.0
        np.testing.assert_allclose(lse[0], st["lse"], atol=1e-5)


def test_tiny_stream():
    wl = synth.WORKLOADS["tiny"]
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl))
    assert r["hits"] > 10


def test_tiny_all_miss_equals_dense():
    wl = synth.WORKLOADS["tiny"]
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tau=0.0)
    assert r["hits"] == 0


def test_llama8b_32k_stream():
    wl = synth.WORKLOADS["llama8b_32k"]
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl))
    assert r["hits"] > 100


@pytest.mark.slow
def test_long_128k_stream_full():
    """The benchmark's workload at full size, every step, in the bench's launch configuration."""
    wl = synth.WORKLOADS["long_128k"]
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl))
    assert r["hits"] > 300


@pytest.mark.slow
def test_long_128k_all_miss_steps():
    wl = synth.WORKLOADS["long_128k"]
    compare_stream(wl, synth.queries(wl, 4), synth.kv_cache(wl, 4), tau=0.0)


@pytest.mark.slow
def test_paged_mixed_stream_full():
    """The paged workload at its stated size: 16 sequences of 8K-64K keys on a
    shuffled pool of 16-key pages, all 64 steps, every step against the oracle."""
    wl = synth.WORKLOADS["paged_mixed"]
    assert wl.steps == 64
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl))
    assert 0 < r["hits"] < wl.steps * wl.B * wl.Hkv


def test_paged_equals_contiguous_bitwise():
    """The same keys in contiguous and paged layouts give identical bits (chunking is by logical key)."""
    wl = synth.WORKLOADS["paged_mixed"].with_(B=4, L0=(3000, 777, 4100, 1601), steps=16)
    stream = synth.queries(wl)
    paged = synth.kv_cache(wl)
    cap = paged.max_seq
    Kc = np.zeros((wl.B, cap, wl.Hkv, wl.D), np.uint16)
    Vc = np.zeros_like(Kc)
    ps = wl.page_size
    for b in range(wl.B):
        n = int(np.sum(paged.block_table[b] >= 0))
        pages = paged.block_table[b, :n]
        Kc[b, :n * ps] = paged.K[pages].reshape(n * ps, wl.Hkv, wl.D)
        Vc[b, :n * ps] = paged.V[pages].reshape(n * ps, wl.Hkv, wl.D)
    contig = synth.KVCache(Kc, Vc, None, cap, 0)
    wc = wl.with_(page_size=0)
    g1 = DeviceRun(wl, paged)
    g2 = DeviceRun(wc, contig)
    for t in range(wl.steps):
        a = g1.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        b = g2.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        for x, y in zip(a, b):
            np.testing.assert_array_equal(x, y)


def _continuous_append_stream(wl, steps):
    """Paged cache filled one row per step through mac_append_kv (every decode
    row poisoned with NaN until its append), the window updated every step;
    every step against the oracle.  Returns the number of hits."""
    import kv_cache_reuse_b200 as mac
    stream = synth.queries(wl, steps)
    cache = synth.kv_cache(wl, steps)
    torch, dev = torch_dev()
    Kd = torch.from_numpy(cache.K.view(np.int16)).to(dev)
    Vd = torch.from_numpy(cache.V.view(np.int16)).to(dev)
    ps = wl.page_size
    pos = np.concatenate([np.arange(wl.L0[b], wl.L0[b] + steps) for b in range(wl.B)])
    seq = np.repeat(np.arange(wl.B), steps)
    pg = torch.from_numpy(cache.block_table[seq, pos // ps].astype(np.int64)).to(dev)
    row = torch.from_numpy((pos % ps).astype(np.int64)).to(dev)
    Kd[pg, row] = 0x7FC0
    Vd[pg, row] = 0x7FC0
    gpu = DeviceRun(wl, cache, K_dev=Kd, V_dev=Vd)
    orc = oracle.Oracle.for_workload(wl, cache)
    knew = torch.empty((wl.B, wl.Hkv, wl.D), dtype=torch.int16, device=dev)
    vnew = torch.empty_like(knew)
    hits = 0
    for t in range(steps):
        kr, vr = synth.step_rows(cache, stream.seq_lens[t])
        knew.copy_(torch.from_numpy(kr.view(np.int16)))
        vnew.copy_(torch.from_numpy(vr.view(np.int16)))
        gpu.lens.copy_(torch.from_numpy(stream.seq_lens[t]))
        mac.mac_append_kv(gpu.st, Kd, Vd, gpu.bt, gpu.lens, knew, vnew)
        r = orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, cache.block_table, stream.seq_lens[t])
        out, lse, hit, mpos = gpu.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        np.testing.assert_array_equal(hit, r.hit, err_msg="hit mask, step %d" % t)
        np.testing.assert_array_equal(mpos, r.match_pos, err_msg="match position, step %d" % t)
        assert np.abs(out - r.out).max() <= OUT_TOL, "out, step %d" % t
        assert np.abs(lse - r.lse).max() <= LSE_TOL, "lse, step %d" % t
        hits += int(hit.sum())
    assert gpu.st.get_status() == 0
    return hits


def test_continuous_append_stream():
    """The first 96 steps of the continuous workload."""
    wl = synth.WORKLOADS["continuous_16k"]
    assert _continuous_append_stream(wl, 96) > 0


@pytest.mark.slow
def test_continuous_append_stream_full():
    """The continuous workload at its stated size: 8 sequences, 16K prefix,
    all 4096 decode steps with an append each step, hits from the two-state
    Markov chain -- the ring, the hit chains and the append path over a long run."""
    wl = synth.WORKLOADS["continuous_16k"]
    assert wl.steps == 4096
    hits = _continuous_append_stream(wl, wl.steps)
    assert 0.6 * wl.steps * wl.B * wl.Hkv < hits < wl.steps * wl.B * wl.Hkv


def test_ring_state_matches_oracle_window():
    import kv_cache_reuse_b200 as mac
    wl = synth.WORKLOADS["tiny"].with_(steps=40)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    r = compare_stream(wl, stream, cache)
    gpu, orc = r["gpu"], r["oracle"]
    st = mac.parse_state(gpu.st.export_state(), wl.W, wl.G, wl.D)
    W1 = wl.W + 1
    n = int(st["steps"][0])
    assert n == wl.steps
    q_o, o_o, m_o, l_o, pos_o = orc.window(0)
    for age in range(wl.W):  # oracle window is oldest first
        slot = (n - 1 - age) % W1
        e = len(pos_o) - 1 - age
        assert st["pos"][0, slot] == pos_o[e]
        np.testing.assert_array_equal(st["q"][0, slot], q_o[e])
        np.testing.assert_allclose(st["o"][0, slot], o_o[e], atol=OUT_TOL)
        lse_g = st["m"][0, slot] + np.log(st["l"][0, slot])
        np.testing.assert_allclose(lse_g, m_o[e] + np.log(l_o[e]), atol=LSE_TOL)


def test_export_import_resumes_identically():
    import kv_cache_reuse_b200 as mac
    wl = synth.WORKLOADS["tiny"].with_(steps=30)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    a = DeviceRun(wl, cache)
    for t in range(15):
        a.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
    buf = a.st.export_state()
    b = DeviceRun(wl, cache)
    b.st.import_state(buf)
    for t in range(15, 30):
        x = a.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        y = b.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        for u, v in zip(x, y):
            np.testing.assert_array_equal(u, v)


def test_host_entry_matches_device_entry():
    import kv_cache_reuse_b200 as mac
    wl = synth.WORKLOADS["tiny"].with_(steps=20)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    a = DeviceRun(wl, cache)
    b = DeviceRun(wl, cache)
    torch = a.torch
    out_h = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.float32).pin_memory()
    lse_h = torch.empty((wl.B, wl.Hq), dtype=torch.float32).pin_memory()
    hit_h = torch.empty((wl.B, wl.Hkv), dtype=torch.uint8).pin_memory()
    mp_h = torch.empty((wl.B, wl.Hkv), dtype=torch.int32).pin_memory()
    for t in range(wl.steps):
        x = a.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        q_h = torch.from_numpy(stream.q[t]).pin_memory()
        p_h = torch.from_numpy(stream.rope_pos[t]).pin_memory()
        l_h = torch.from_numpy(stream.seq_lens[t]).pin_memory()
        rc = mac.mac_decode_step_host(b.st, q_h, p_h, l_h, None, None, b.K, b.V, None, out_h, lse_h, hit_h, mp_h)
        assert rc == mac.MAC_OK
        for u, v in zip(x, (out_h.numpy(), lse_h.numpy(), hit_h.numpy(), mp_h.numpy())):
            np.testing.assert_array_equal(u, v)


def test_host_entry_append_recapture():
    """Host entry with appends on a paged pool, a swap of the cache buffers and a
    work-split change mid-stream (each forces a new recording), against the device
    entry on the same inputs, bit for bit."""
    import kv_cache_reuse_b200 as mac
    wl = synth.WORKLOADS["continuous_16k"].with_(L0=(3000, 1777, 4100, 2601), B=4)
    steps = 30
    stream = synth.queries(wl, steps)
    cache = synth.kv_cache(wl, steps)
    torch, dev = torch_dev()
    pool = [torch.from_numpy(x.view(np.int16)).to(dev) for x in (cache.K, cache.V)]
    a = DeviceRun(wl, cache, K_dev=pool[0].clone(), V_dev=pool[1].clone())
    b = DeviceRun(wl, cache, K_dev=pool[0].clone(), V_dev=pool[1].clone())
    Kb2, Vb2 = b.K.clone(), b.V.clone()
    knew = torch.empty((wl.B, wl.Hkv, wl.D), dtype=torch.int16, device=dev)
    vnew = torch.empty_like(knew)
    out_h = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.float32)
    lse_h = torch.empty((wl.B, wl.Hq), dtype=torch.float32)
    hit_h = torch.empty((wl.B, wl.Hkv), dtype=torch.uint8)
    mp_h = torch.empty((wl.B, wl.Hkv), dtype=torch.int32)
    Kb, Vb = b.K, b.V
    hits = 0
    for t in range(steps):
        kr, vr = synth.step_rows(cache, stream.seq_lens[t])
        knew.copy_(torch.from_numpy(kr.view(np.int16)))
        vnew.copy_(torch.from_numpy(vr.view(np.int16)))
        a.lens.copy_(torch.from_numpy(stream.seq_lens[t]))
        mac.mac_append_kv(a.st, a.K, a.V, a.bt, a.lens, knew, vnew)
        x = a.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        if t == 10:  # move the cache to other buffers: the recording must follow
            Kb2.copy_(Kb)
            Vb2.copy_(Vb)
            torch.cuda.synchronize()
            Kb, Vb = Kb2, Vb2
        if t == 20:  # a work-split change drops the recording
            mac.mac_set_piece_cost(b.st, 512)
            mac.mac_set_piece_cost(a.st, 512)
        kh = torch.from_numpy(kr.view(np.int16).copy())
        vh = torch.from_numpy(vr.view(np.int16).copy())
        rc = mac.mac_decode_step_host(b.st, torch.from_numpy(stream.q[t]), torch.from_numpy(stream.rope_pos[t]),
                                      torch.from_numpy(stream.seq_lens[t]), kh, vh, Kb, Vb, b.bt, out_h, lse_h,
                                      hit_h, mp_h)
        assert rc == mac.MAC_OK
        for u, v in zip(x, (out_h.numpy(), lse_h.numpy(), hit_h.numpy(), mp_h.numpy())):
            np.testing.assert_array_equal(u, v, err_msg="step %d" % t)
        hits += int(x[2].sum())
    assert hits > 0 and hits < steps * wl.B * wl.Hkv
    assert a.st.get_status() == 0 and b.st.get_status() == 0


@pytest.mark.parametrize("case", ["one_key", "band0", "window1", "ragged", "full_capacity", "band_covers", "d128_short",
                                  "window_max", "many_units", "page64"])
def test_edge_cases(case):
    base = synth.WORKLOADS["tiny"]
    kw = {}
    if case == "one_key":
        kw = dict(L0=(0,), steps=12)  # first step sees a single key
    elif case == "band0":
        kw = dict(band=0, steps=32)
    elif case == "window1":
        kw = dict(W=1, steps=32)
    elif case == "ragged":
        kw = dict(L0=(1013,), steps=20)
    elif case == "full_capacity":
        kw = dict(L0=(500,), steps=12)
    elif case == "band_covers":
        kw = dict(L0=(40,), band=500, steps=24)
    elif case == "d128_short":
        base = synth.WORKLOADS["llama8b_32k"]
        kw = dict(L0=(37,), steps=40, W=8)
    elif case == "window_max":  # the largest window: the match kernel scans its slots in several batches
        kw = dict(L0=(60,), steps=280, W=256, band=16)
    elif case == "many_units":  # 160 units: 320 work items, more than one pass of the plan build
        kw = dict(B=40, Hq=16, Hkv=4, L0=tuple(200 + 37 * i for i in range(40)), steps=6)
    elif case == "page64":  # 64-key pages: several boxes per page, block table over a shuffled pool
        base = synth.WORKLOADS["paged_mixed"]
        kw = dict(B=3, L0=(3000, 700, 2100), steps=12, page_size=64)
    wl = base.with_(**kw)
    stream = synth.queries(wl)
    cache = synth.kv_cache(wl)  # capacity = L0 + steps exactly: the last step fills it
    compare_stream(wl, stream, cache)


def test_weighted_split_all_miss():
    """Large all-miss steps take the rate-weighted split (ranges sized by each
    SM's learned rate, taken by the CTA on that SM); results match the oracle
    on the first step (even weights) and the later ones (learned weights)."""
    wl = synth.WORKLOADS["llama8b_32k"].with_(B=4, L0=(32768, 30000, 31000, 29000), steps=5)
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tau=0.0)
    assert r["hits"] == 0


def test_reproducible_split_gives_identical_bits():
    """mac_set_reproducible: on large steps (above the rate-weighted split's
    threshold) two states with different histories -- one first ran steps of
    another stream, which would have taught it per-SM rates -- give the same
    bits on the same inputs, and match the oracle."""
    import kv_cache_reuse_b200 as mac
    wl = synth.WORKLOADS["llama8b_32k"].with_(B=4, L0=(32768, 30000, 31000, 29000), steps=6)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    a = DeviceRun(wl, cache, tune={"reproducible": 1})
    b = DeviceRun(wl, cache, tune={"reproducible": 1})
    other = synth.queries(wl.with_(seed=wl.seed + 99))
    for t in range(4):
        b.step(other.q[t], other.rope_pos[t], other.seq_lens[t])
    for s_ in range(wl.B):
        mac.mac_reset_seq(b.st, s_)
    orc = oracle.Oracle.for_workload(wl, cache)
    for t in range(wl.steps):
        x = a.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        y = b.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        for u, v in zip(x, y):
            np.testing.assert_array_equal(u, v, err_msg="step %d" % t)
        r = orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, cache.block_table, stream.seq_lens[t])
        np.testing.assert_array_equal(x[2], r.hit)
        np.testing.assert_array_equal(x[3], r.match_pos)
        assert float(np.abs(x[0] - r.out).max()) <= OUT_TOL and float(np.abs(x[1] - r.lse).max()) <= LSE_TOL
    assert a.st.get_status() == 0 and b.st.get_status() == 0


def test_one_launch_is_used_where_it_applies():
    """Groups of up to 8 heads with one decision per KV head run the step as
    one launch by default; per-head matching, groups of 16-64 heads and the
    switch mac_set_one_launch(0) run two."""
    import kv_cache_reuse_b200 as mac
    tiny = synth.WORKLOADS["tiny"]
    cache = synth.kv_cache(tiny.with_(steps=2))
    assert mac.mac_one_launch(DeviceRun(tiny, cache).st) == 1
    assert mac.mac_one_launch(DeviceRun(tiny, cache, tune={"one_launch": 0}).st) == 0
    assert mac.mac_one_launch(DeviceRun(tiny, cache, per_head=1).st) == 0
    assert mac.mac_one_launch(DeviceRun(tiny.with_(Hq=32), cache).st) == 0


@pytest.mark.parametrize("case", ["tiny", "llama", "paged", "weighted_all_miss", "many_units", "bf16"])
def test_two_launch_path(case):
    """mac_decode_step with the one-launch step switched off: the match kernel
    (which lays out every unit's items) and the attention kernel launched one
    after the other, against the oracle."""
    tiny, llama, paged = synth.WORKLOADS["tiny"], synth.WORKLOADS["llama8b_32k"], synth.WORKLOADS["paged_mixed"]
    tau, rb = None, 0
    if case == "tiny":
        wl = tiny.with_(steps=40)
    elif case == "llama":
        wl = llama.with_(L0=(9000,), steps=40)
    elif case == "paged":
        wl = paged.with_(B=4, L0=(9000, 1500, 300, 4100), steps=16)
    elif case == "weighted_all_miss":
        wl, tau = llama.with_(B=4, L0=(32768, 30000, 31000, 29000), steps=4), 0.0
    elif case == "many_units":
        wl = tiny.with_(B=40, Hq=16, Hkv=4, L0=tuple(200 + 37 * i for i in range(40)), steps=6)
    else:
        wl, rb = llama.with_(L0=(6000,), steps=24), 1
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tau=tau, ring_bf16=rb, tune={"one_launch": 0})
    assert r["gpu"].st is not None


@pytest.mark.parametrize("one_launch", [1, 0])
def test_trace_counts_keys_and_orders_phases(one_launch):
    """mac_set_trace: the device's count of keys attended with the current
    query equals the keys the oracle reads at every step, and on steps where
    every unit hits it is the same at 8K and 32K keys of context (page 1: the
    cost of a hit does not grow with the context); each CTA's phase times come
    in order."""
    import kv_cache_reuse_b200 as mac
    per_ctx = {}
    for L in (8192, 32768):
        wl = synth.WORKLOADS["llama8b_32k"].with_(B=2, L0=(L, L), steps=10, hit_model=("iid", 1.0))
        stream, cache = synth.queries(wl), synth.kv_cache(wl)
        gpu = DeviceRun(wl, cache, tune={"trace": 1, "one_launch": one_launch})
        orc = oracle.Oracle.for_workload(wl, cache)
        keys = []
        for t in range(wl.steps):
            r = orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, cache.block_table, stream.seq_lens[t])
            out, lse, hit, mpos = gpu.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
            np.testing.assert_array_equal(hit, r.hit)
            assert float(np.abs(out - r.out).max()) <= OUT_TOL
            stamps, counters = mac.mac_get_trace(gpu.st)
            assert int(counters[0]) == r.keys_read, "step %d" % t
            assert int(counters[1]) >= 1 and int(counters[2]) + int(counters[3]) >= 1
            keys.append((int(r.hit.all()), int(counters[0])))
            for row in stamps.astype(np.int64):
                seen = [row[k] for k in (0, 1, 2, 3, 4, 7, 9, 10, 11) if row[k] > 0]
                assert seen == sorted(seen), row
                if row[8] > 0:  # the laying-out CTA published the table after its ticket
                    assert row[4] <= row[8] and (row[9] == 0 or row[8] <= row[9])
            assert (stamps[:, 0] > 0).any()
        per_ctx[L] = keys
        assert gpu.st.get_status() == 0
    hit_steps = [t for t in range(1, 10) if per_ctx[8192][t][0] and per_ctx[32768][t][0]]
    assert len(hit_steps) >= 5
    for t in hit_steps:
        assert per_ctx[8192][t][1] == per_ctx[32768][t][1], t


_SPLIT = {"whole_unit_keys": 0, "piece_cost": 0, "min_keys_per_cta": 64}


@pytest.mark.parametrize("case", ["g1_d64", "g1_d128_paged", "g2_split", "g3_paged", "g5_d64", "g6_split",
                                  "g7_paged", "g8_d64", "g8_d128", "g8_split"])
def test_group_sizes(case):
    """Groups of 1 to 8 query heads per KV head (multi-head attention to
    8-way GQA), whole and split units, contiguous and paged KV."""
    tiny, llama, paged = synth.WORKLOADS["tiny"], synth.WORKLOADS["llama8b_32k"], synth.WORKLOADS["paged_mixed"]
    tune = None
    if case == "g1_d64":
        wl = tiny.with_(Hq=2, Hkv=2, steps=40)
    elif case == "g1_d128_paged":
        wl = paged.with_(B=2, Hq=8, Hkv=8, L0=(3000, 700), steps=16)
    elif case == "g2_split":
        wl, tune = tiny.with_(Hq=4, Hkv=2, steps=40), _SPLIT
    elif case == "g3_paged":
        wl = paged.with_(B=3, Hq=12, Hkv=4, L0=(2500, 900, 4100), steps=16)
    elif case == "g5_d64":
        wl = tiny.with_(Hq=10, Hkv=2, steps=40)
    elif case == "g6_split":
        wl, tune = llama.with_(B=2, Hq=12, Hkv=2, L0=(5000, 3100), steps=16), _SPLIT
    elif case == "g7_paged":  # 28 query heads over 4 KV heads
        wl = paged.with_(B=3, Hq=28, Hkv=4, L0=(3000, 1200, 6000), steps=16)
    elif case == "g8_d64":
        wl = tiny.with_(Hq=8, Hkv=1, steps=40)
    elif case == "g8_d128":  # 64 query heads over 8 KV heads
        wl = llama.with_(B=2, Hq=64, Hkv=8, L0=(9000, 4000), steps=24)
    else:
        wl, tune = llama.with_(B=2, Hq=16, Hkv=2, L0=(6000, 2000), steps=16), _SPLIT
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tune=tune)
    assert r["hits"] > 0


@pytest.mark.parametrize("case", ["g16_d128", "g32_mqa", "g64_mqa", "g16_d64", "g64_d64", "g32_paged", "g64_bf16",
                                  "g32_cut1", "g16_band_covers", "g32_window_max"])
def test_mqa_groups(case):
    """Groups of 16, 32 and 64 query heads per KV head (multi-query attention,
    which page 1 says the method composes with): the heads run in chunks of 8
    over the same K/V boxes, the window scan over G/8 CTAs per unit; decisions
    bit-exact, outputs within tolerance, every step, hits and misses."""
    tiny, llama, paged = synth.WORKLOADS["tiny"], synth.WORKLOADS["llama8b_32k"], synth.WORKLOADS["paged_mixed"]
    cut, qb, rb = 0, 0, 0
    if case == "g16_d128":
        wl = llama.with_(B=2, Hq=32, Hkv=2, L0=(5000, 3100), steps=16)
    elif case == "g32_mqa":
        wl = llama.with_(B=2, Hq=32, Hkv=1, L0=(9000, 4000), steps=24)
    elif case == "g64_mqa":
        wl = llama.with_(B=1, Hq=64, Hkv=1, L0=(12000,), steps=24)
    elif case == "g16_d64":
        wl = tiny.with_(Hq=16, Hkv=1, steps=40)
    elif case == "g64_d64":
        wl = tiny.with_(B=2, Hq=64, Hkv=1, L0=(1500, 700), steps=24)
    elif case == "g32_paged":
        wl = paged.with_(B=3, Hq=32, Hkv=1, L0=(3000, 1200, 6000), steps=16)
    elif case == "g64_bf16":  # bf16 queries and window
        wl, qb, rb = llama.with_(B=2, Hq=64, Hkv=1, L0=(6000, 2500), steps=16), 1, 1
    elif case == "g32_cut1":
        wl, cut = llama.with_(B=2, Hq=32, Hkv=1, L0=(3000, 5000), steps=16), 1
    elif case == "g16_band_covers":  # the band reaches key 0: every reused prefix is empty
        wl = tiny.with_(Hq=16, Hkv=1, L0=(40,), band=500, steps=24)
    else:  # the largest window: the chunk CTAs scan their slots in several batches
        wl = tiny.with_(Hq=32, Hkv=1, L0=(60,), steps=280, W=256, band=16)
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), cut_mode=cut, q_bf16=qb, ring_bf16=rb)
    assert 0 < r["hits"] < wl.steps * wl.B * wl.Hkv


@pytest.mark.parametrize("Hq,Hkv,L0", [(32, 1, (32768, 20000)), (64, 1, (24000, 30000)), (64, 4, (32768, 9000))])
def test_mqa_all_miss_large(Hq, Hkv, L0):
    """Large all-miss steps of multi-query groups: the rate-weighted split, a
    single KV head's keys cut over every CTA (more than 100 partials per unit,
    merged chunk by chunk)."""
    wl = synth.WORKLOADS["llama8b_32k"].with_(B=2, Hq=Hq, Hkv=Hkv, L0=L0, steps=3)
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tau=0.0)
    assert r["hits"] == 0


def test_mqa_export_matches_oracle_window():
    """The window of a 32-head group after a stream: positions and queries
    equal to the oracle's, stored states within tolerance."""
    import kv_cache_reuse_b200 as mac
    wl = synth.WORKLOADS["tiny"].with_(Hq=32, Hkv=1, steps=30)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    r = compare_stream(wl, stream, cache)
    st = mac.parse_state(r["gpu"].st.export_state(), wl.W, wl.G, wl.D)
    q, o, m, l, pos = r["oracle"].window(0)
    n = len(pos)
    slots = [(wl.steps - n + i) % (wl.W + 1) for i in range(n)]
    np.testing.assert_array_equal(st["pos"][0, slots], pos)
    np.testing.assert_array_equal(st["q"][0, slots], q)
    np.testing.assert_allclose(st["o"][0, slots], o, atol=OUT_TOL)
    np.testing.assert_allclose(st["m"][0, slots] + np.log(st["l"][0, slots]), m + np.log(l), atol=LSE_TOL)


@pytest.mark.parametrize("G,B,L0,band", [(16, 3, (40, 130, 300), 64), (64, 2, (100, 700), 600), (32, 2, (127, 129), 16)])
def test_mqa_tensor_memory_edges(G, B, L0, band):
    """The tensor-memory path (head dim 128) at its edges: sequences shorter
    than one 128-key tile or just across it, bands that reach key 0 (empty
    reused prefix, empty amend range), pieces that start and end inside a
    tile -- decisions bit-exact and outputs within tolerance at every step."""
    wl = synth.WORKLOADS["llama8b_32k"].with_(B=B, Hq=G, Hkv=1, L0=L0, band=band, steps=20)
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl))
    assert r["hits"] > 0


def test_mqa_steps_repeat_bit_for_bit():
    """The tensor-memory path of a 32-head group on large all-miss steps (a
    single KV head's keys cut over every CTA) and on the repeats after them:
    two states fed the same stream give the same bits (each partial comes from
    one range of the split whichever CTA runs it, and the merge folds them in a
    fixed order), and both match the oracle."""
    wl = synth.WORKLOADS["llama8b_32k"].with_(B=2, Hq=32, Hkv=1, L0=(32768, 20000), steps=5)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    a, b = DeviceRun(wl, cache), DeviceRun(wl, cache)
    orc = oracle.Oracle.for_workload(wl, cache)
    for t in range(wl.steps):
        x = a.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        y = b.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        for u, v in zip(x, y):
            np.testing.assert_array_equal(u, v, err_msg="step %d" % t)
        r = orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, cache.block_table, stream.seq_lens[t])
        np.testing.assert_array_equal(x[2], r.hit)
        np.testing.assert_array_equal(x[3], r.match_pos)
        assert float(np.abs(x[0] - r.out).max()) <= OUT_TOL and float(np.abs(x[1] - r.lse).max()) <= LSE_TOL
    assert a.st.get_status() == 0 and b.st.get_status() == 0


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (24, 8), (64, 8)])
def test_group_sizes_all_miss_large(Hq, Hkv):
    """Large all-miss steps (weighted split, many partials per unit) for
    groups of 1, 3 and 8."""
    wl = synth.WORKLOADS["llama8b_32k"].with_(B=2, Hq=Hq, Hkv=Hkv, L0=(32768, 20000), steps=3)
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tau=0.0)
    assert r["hits"] == 0


@pytest.mark.parametrize("G", [1, 4, 16, 64])
def test_threshold_is_strict_and_ties_pick_the_most_recent(G):
    """Decisions at the edges the generator's margins stay away from: a
    distance exactly at the threshold misses and one ulp more of threshold
    hits (the queries make the distance exactly 0.25 in fp32 and fp64), and
    equal distances pick the most recent entry -- the kernels decide as the
    oracle does."""
    wl = synth.WORKLOADS["tiny"].with_(Hq=G, Hkv=1, steps=6)
    cache, stream = synth.kv_cache(wl), synth.queries(wl)
    q0 = ((np.arange(G * wl.D).reshape(1, G, wl.D) % 16 - 8) / 8).astype(np.float32)
    q1 = q0.copy()
    q1[0, :, 3] += np.float32(0.5)
    far = (q0 + np.float32(3.0)).astype(np.float32)
    for tau, hit1 in ((0.25, 0), (float(np.nextafter(np.float32(0.25), np.float32(1.0))), 1)):
        gpu = DeviceRun(wl, cache, tau=tau)
        orc = oracle.Oracle.for_workload(wl, cache, tau=tau)
        for t, qt in enumerate([q0, q1, far, q0, q0]):
            r = orc.step(qt, stream.rope_pos[t], cache.K, cache.V, cache.block_table, stream.seq_lens[t])
            out, lse, hit, mpos = gpu.step(qt, stream.rope_pos[t], stream.seq_lens[t])
            np.testing.assert_array_equal(hit, r.hit, err_msg="tau %r step %d" % (tau, t))
            np.testing.assert_array_equal(mpos, r.match_pos, err_msg="tau %r step %d" % (tau, t))
            assert float(np.abs(out - r.out).max()) <= OUT_TOL and float(np.abs(lse - r.lse).max()) <= LSE_TOL
            if t == 1:
                assert int(hit[0, 0]) == hit1
            if t == 4:  # steps 0 and 3 hold the same query: the later one is reused
                assert hit[0, 0] == 1 and mpos[0, 0] == stream.seq_lens[3][0] - 1
        assert gpu.st.get_status() == 0


@pytest.mark.parametrize("case", ["g4_d128", "g8_d128", "g3_d64", "g8_d128_hits"])
def test_one_unit_over_every_cta(case):
    """A single (sequence, KV head) whose keys are cut over all 148 CTAs: the
    merge folds ~150 partials, several rounds of loads per warp, with the
    group padded (3 of 4) or exact (4, 8), on misses and on hits (the reused
    state joins segment A, the amend band and tail are the fresh range)."""
    tiny, llama = synth.WORKLOADS["tiny"], synth.WORKLOADS["llama8b_32k"]
    tau = 0.0
    if case == "g4_d128":
        wl = llama.with_(B=1, Hq=4, Hkv=1, L0=(40000,), steps=3)
    elif case == "g8_d128":
        wl = llama.with_(B=1, Hq=8, Hkv=1, L0=(24000,), steps=3)
    elif case == "g3_d64":
        wl = tiny.with_(B=1, Hq=3, Hkv=1, L0=(30000,), steps=3)
    else:
        wl, tau = llama.with_(B=1, Hq=8, Hkv=1, L0=(24000,), steps=12), None
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tau=tau, tune={"whole_unit_keys": 0})
    assert r["hits"] == 0 if tau == 0.0 else r["hits"] > 0


@pytest.mark.parametrize("case", ["g4_d64", "g4_d128", "g4_split", "g3_paged", "g8_split", "g1", "g6_cut1"])
def test_per_head_matching(case):
    """Per-head matching on streams whose heads repeat on their own: every
    head's decision bit-exact, ragged reuse boundaries inside a group (each
    head masked to its own range of the amend band), each head's state from
    its own ring slot, whole and split units."""
    tiny, llama, paged = synth.WORKLOADS["tiny"], synth.WORKLOADS["llama8b_32k"], synth.WORKLOADS["paged_mixed"]
    tune, cut = None, 0
    if case == "g4_d64":
        wl = tiny.with_(head_labels=True, steps=48)
    elif case == "g4_d128":
        wl = llama.with_(head_labels=True, L0=(6000,), steps=32)
    elif case == "g4_split":
        wl, tune = tiny.with_(head_labels=True, steps=40), _SPLIT
    elif case == "g3_paged":
        wl = paged.with_(B=3, Hq=12, Hkv=4, L0=(2500, 900, 4100), steps=16, head_labels=True)
    elif case == "g8_split":
        wl, tune = llama.with_(B=2, Hq=16, Hkv=2, L0=(6000, 2000), steps=16, head_labels=True), _SPLIT
    elif case == "g1":
        wl = tiny.with_(Hq=2, Hkv=2, head_labels=True, steps=32)
    else:
        wl, cut = llama.with_(B=2, Hq=12, Hkv=2, L0=(3000, 5000), steps=16, head_labels=True), 1
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tune=tune, cut_mode=cut, per_head=1)
    hits = r["hits"]
    assert 0 < hits < wl.steps * wl.B * wl.Hq


def test_bf16_host_entry_matches_device_entry():
    """The host entry with bf16 queries (its input block carries 2 bytes per
    query element) and a bf16 window, against the device entry, bit for bit."""
    import kv_cache_reuse_b200 as mac
    wl = synth.WORKLOADS["tiny"].with_(steps=20)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    a = DeviceRun(wl, cache, q_bf16=1, ring_bf16=1)
    b = DeviceRun(wl, cache, q_bf16=1, ring_bf16=1)
    torch = a.torch
    out_h = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.float32).pin_memory()
    lse_h = torch.empty((wl.B, wl.Hq), dtype=torch.float32).pin_memory()
    hit_h = torch.empty((wl.B, wl.Hkv), dtype=torch.uint8).pin_memory()
    mp_h = torch.empty((wl.B, wl.Hkv), dtype=torch.int32).pin_memory()
    hits = 0
    for t in range(wl.steps):
        x = a.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        q_h = torch.from_numpy(synth.f32_to_bf16_bits(stream.q[t]).view(np.int16)).pin_memory()
        p_h = torch.from_numpy(stream.rope_pos[t]).pin_memory()
        l_h = torch.from_numpy(stream.seq_lens[t]).pin_memory()
        rc = mac.mac_decode_step_host(b.st, q_h, p_h, l_h, None, None, b.K, b.V, None, out_h, lse_h, hit_h, mp_h)
        assert rc == mac.MAC_OK
        for u, v in zip(x, (out_h.numpy(), lse_h.numpy(), hit_h.numpy(), mp_h.numpy())):
            np.testing.assert_array_equal(u, v)
        hits += int(x[2].sum())
    assert hits > 0


def test_per_head_weighted_split():
    """Per-head matching on large steps (most units have a head that misses, so
    they read every key): the rate-weighted split with per-head key bounds."""
    wl = synth.WORKLOADS["llama8b_32k"].with_(B=4, L0=(32768, 30000, 31000, 29000), steps=6, head_labels=True,
                                              hit_model=("iid", 0.5))
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), per_head=1)
    assert 0 < r["hits"] < wl.steps * wl.B * wl.Hq


def test_per_head_host_entry_matches_device_entry():
    """The host entry returns [B][Hq] decisions with per-head matching."""
    import kv_cache_reuse_b200 as mac
    wl = synth.WORKLOADS["tiny"].with_(steps=20, head_labels=True)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    a = DeviceRun(wl, cache, per_head=1)
    b = DeviceRun(wl, cache, per_head=1)
    torch = a.torch
    out_h = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.float32).pin_memory()
    lse_h = torch.empty((wl.B, wl.Hq), dtype=torch.float32).pin_memory()
    hit_h = torch.empty((wl.B, wl.Hq), dtype=torch.uint8).pin_memory()
    mp_h = torch.empty((wl.B, wl.Hq), dtype=torch.int32).pin_memory()
    for t in range(wl.steps):
        x = a.step(stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        q_h = torch.from_numpy(stream.q[t]).pin_memory()
        p_h = torch.from_numpy(stream.rope_pos[t]).pin_memory()
        l_h = torch.from_numpy(stream.seq_lens[t]).pin_memory()
        rc = mac.mac_decode_step_host(b.st, q_h, p_h, l_h, None, None, b.K, b.V, None, out_h, lse_h, hit_h, mp_h)
        assert rc == mac.MAC_OK
        for u, v in zip(x, (out_h.numpy(), lse_h.numpy(), hit_h.numpy(), mp_h.numpy())):
            np.testing.assert_array_equal(u, v)


@pytest.mark.parametrize("case", ["tiny", "llama", "split", "g3_paged", "g8", "per_head", "q_only", "q_and_ring",
                                  "q_paged_per_head"])
def test_bf16_window_and_queries(case):
    """bf16 window (queries and stored outputs rounded to bf16, as the oracle
    does) and bf16 query input, alone and together, over the kernel variants."""
    tiny, llama, paged = synth.WORKLOADS["tiny"], synth.WORKLOADS["llama8b_32k"], synth.WORKLOADS["paged_mixed"]
    tune, ph, qb, rb = None, 0, 0, 1
    if case == "tiny":
        wl = tiny.with_(steps=48)
    elif case == "llama":
        wl = llama.with_(L0=(6000,), steps=48)
    elif case == "split":
        wl, tune = tiny.with_(steps=40), _SPLIT
    elif case == "g3_paged":
        wl = paged.with_(B=3, Hq=12, Hkv=4, L0=(2500, 900, 4100), steps=16)
    elif case == "g8":
        wl = llama.with_(B=2, Hq=64, Hkv=8, L0=(9000, 4000), steps=16)
    elif case == "per_head":
        wl, ph = tiny.with_(head_labels=True, steps=40), 1
    elif case == "q_only":
        wl, qb, rb = llama.with_(L0=(6000,), steps=32), 1, 0
    elif case == "q_and_ring":
        wl, qb = tiny.with_(steps=40), 1
    else:
        wl, qb, ph = paged.with_(B=3, Hq=8, Hkv=2, L0=(2500, 900, 4100), steps=16, head_labels=True), 1, 1
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tune=tune, per_head=ph, q_bf16=qb, ring_bf16=rb)
    assert r["hits"] > 0


def test_bf16_window_export_matches_oracle_window():
    """The exported bf16 window: queries bit-equal to the rounded inputs; the
    stored outputs (bf16 bits) within the output tolerance of the oracle's
    rounded ones, as for the fp32 window (rounding to neighbouring bf16 values
    can carry along chains of hits)."""
    import kv_cache_reuse_b200 as mac
    wl = synth.WORKLOADS["tiny"].with_(steps=24)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    r = compare_stream(wl, stream, cache, ring_bf16=1)
    st = mac.parse_state(r["gpu"].st.export_state(), wl.W, wl.G, wl.D)
    assert st["q"].dtype == np.uint16 and st["o"].dtype == np.uint16
    q, o, m, l, pos = r["oracle"].window(0)
    n = len(pos)
    W1 = wl.W + 1
    slots = [(wl.steps - n + i) % W1 for i in range(n)]  # entry of step k sits in slot k mod (W+1)
    np.testing.assert_array_equal(st["q"][0, slots], synth.f32_to_bf16_bits(q))
    np.testing.assert_allclose(synth.bf16_bits_to_f32(st["o"][0, slots]), o, rtol=0, atol=OUT_TOL)
    np.testing.assert_array_equal(st["pos"][0, slots], pos)


@pytest.mark.parametrize("case", ["tiny", "split", "band0", "llama_paged"])
def test_cut_mode_band_ends_at_position(case):
    """cut_mode 1: the stored prefix ends at max(0, p + 1 - band) on both sides."""
    if case == "tiny":
        wl, tune = synth.WORKLOADS["tiny"].with_(steps=40), None
    elif case == "split":  # every range cut over CTAs and merged
        wl, tune = synth.WORKLOADS["tiny"].with_(steps=40), {"whole_unit_keys": 0, "piece_cost": 0,
                                                             "min_keys_per_cta": 64}
    elif case == "band0":  # the prefix covers the current key: an empty tail
        wl, tune = synth.WORKLOADS["tiny"].with_(steps=24, band=0), None
    else:
        wl, tune = synth.WORKLOADS["paged_mixed"].with_(B=3, L0=(3000, 900, 5000), steps=12), None
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tune=tune, cut_mode=1)
    assert r["hits"] > 0


@pytest.mark.parametrize("case", ["tiny", "paged", "per_head_bf16"])
def test_warm_start_from_prefill_then_decode(case):
    """Windows seeded from the first n positions of the stream (as prefill
    positions), then decoding: decisions bit-exact and outputs within tolerance
    of the oracle doing the same, and the seeded ring equal to its window."""
    import kv_cache_reuse_b200 as mac
    ph = qb = rb = 0
    if case == "tiny":
        wl, n = synth.WORKLOADS["tiny"].with_(steps=40), 16
    elif case == "paged":
        wl, n = synth.WORKLOADS["paged_mixed"].with_(B=3, L0=(3000, 900, 5000), steps=20), 8
    else:  # per-head matching, bf16 queries and bf16 window
        wl, n = synth.WORKLOADS["tiny"].with_(steps=40, head_labels=True), 16
        ph = qb = rb = 1
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    if qb:  # the queries as bf16 values: the library reads their bits, the oracle their values
        stream = synth.QueryStream(q=synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(stream.q)), label=stream.label,
                                   src=stream.src, rope_pos=stream.rope_pos, seq_lens=stream.seq_lens)
    gpu = DeviceRun(wl, cache, per_head=ph, q_bf16=qb, ring_bf16=rb)
    orc = oracle.Oracle.for_workload(wl, cache, per_head=ph, ring_bf16=rb)
    torch = gpu.torch
    qh = synth.f32_to_bf16_bits(stream.q[:n]).view(np.int16) if qb else np.ascontiguousarray(stream.q[:n])
    qn = torch.from_numpy(np.ascontiguousarray(qh)).to(gpu.dev)
    pn = torch.from_numpy(np.ascontiguousarray(stream.rope_pos[:n])).to(gpu.dev)
    ln = torch.from_numpy(np.ascontiguousarray(stream.seq_lens[:n])).to(gpu.dev)
    mac.mac_warm_start(gpu.st, n, qn, pn, gpu.K, gpu.V, gpu.bt, ln)
    orc.warm_start(stream.q[:n], stream.rope_pos[:n], cache.K, cache.V, cache.block_table, stream.seq_lens[:n])
    torch.cuda.synchronize()
    st = mac.parse_state(gpu.st.export_state(), wl.W, wl.G, wl.D)
    W1 = wl.W + 1
    for u in range(wl.B * wl.Hkv):
        assert int(st["steps"][u]) == n
        q_o, o_o, m_o, l_o, pos_o = orc.window(u)
        for j in range(n):
            slot = j % W1
            assert st["pos"][u, slot] == pos_o[j]
            if rb:  # the window holds bf16 bits
                np.testing.assert_array_equal(st["q"][u, slot], synth.f32_to_bf16_bits(q_o[j]))
                np.testing.assert_allclose(synth.bf16_bits_to_f32(st["o"][u, slot]), o_o[j], atol=OUT_TOL)
            else:
                np.testing.assert_array_equal(st["q"][u, slot], q_o[j])
                np.testing.assert_allclose(st["o"][u, slot], o_o[j], atol=OUT_TOL)
    r = compare_stream(wl, stream, cache, gpu=gpu, orc=orc, start=n, q_bf16=qb)
    assert r["hits"] > 0


def test_graph_captured_mqa_loop():
    """Two layers of 32 query heads over one KV head (head_dim 128: the
    tensor-memory products and their merge, two launches with programmatic
    dependent launch) recorded as one CUDA graph and replayed for every token:
    each layer against its own fp64 oracle and bit-equal to eager steps."""
    import kv_cache_reuse_b200 as mac
    torch, dev = torch_dev()
    llama = synth.WORKLOADS["llama8b_32k"]
    wls = [llama.with_(B=2, Hq=32, Hkv=1, L0=(3000, 1200), steps=12, seed=20 + l) for l in range(2)]
    streams = [synth.queries(w) for w in wls]
    caches = [synth.kv_cache(w) for w in wls]
    oracles = [oracle.Oracle.for_workload(w, c) for w, c in zip(wls, caches)]
    eager = [DeviceRun(w, c) for w, c in zip(wls, caches)]
    graph = [DeviceRun(w, c) for w, c in zip(wls, caches)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for r in graph:
            mac.mac_decode_step(r.st, r.q, r.pos, r.K, r.V, None, r.lens, r.out, r.lse, r.hit, r.mpos)
    hits = 0
    for t in range(wls[0].steps):
        for l, r in enumerate(graph):
            st = streams[l]
            r.q.copy_(torch.from_numpy(np.ascontiguousarray(st.q[t])))
            r.pos.copy_(torch.from_numpy(st.rope_pos[t]))
            r.lens.copy_(torch.from_numpy(st.seq_lens[t]))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        for l in range(len(graph)):
            st, c = streams[l], caches[l]
            y = (graph[l].out.cpu().numpy(), graph[l].lse.cpu().numpy(), graph[l].hit.cpu().numpy(),
                 graph[l].mpos.cpu().numpy())
            ref = oracles[l].step(st.q[t], st.rope_pos[t], c.K, c.V, c.block_table, st.seq_lens[t])
            np.testing.assert_array_equal(y[2], ref.hit, err_msg="hit mask, layer %d step %d" % (l, t))
            np.testing.assert_array_equal(y[3], ref.match_pos, err_msg="match position, layer %d step %d" % (l, t))
            assert float(np.abs(y[0] - ref.out).max()) <= OUT_TOL, "out, layer %d step %d" % (l, t)
            assert float(np.abs(y[1] - ref.lse).max()) <= LSE_TOL, "lse, layer %d step %d" % (l, t)
            x = eager[l].step(st.q[t], st.rope_pos[t], st.seq_lens[t])
            for u, v in zip(x, y):
                np.testing.assert_array_equal(u, v, err_msg="graph vs eager, layer %d step %d" % (l, t))
            hits += int(ref.hit.sum())
    assert hits > 0
    assert all(r.st.get_status() == 0 for r in graph + eager)


@pytest.mark.parametrize("opts", [{}, {"per_head": 1, "ring_bf16": 1}])
def test_graph_captured_multilayer_loop(opts):
    """Several layers' steps recorded once as one CUDA graph and replayed for
    every token (inputs copied into fixed buffers before each replay): each
    layer's decisions bit-exact and its out / lse within tolerance of its own
    fp64 oracle at every token (also with per-head matching and a bf16 window),
    and the replayed bits equal to the same steps run eagerly."""
    import kv_cache_reuse_b200 as mac
    torch, dev = torch_dev()
    L = 3
    wls = [synth.WORKLOADS["tiny"].with_(steps=24, seed=10 + l, head_labels=bool(opts)) for l in range(L)]
    streams = [synth.queries(w) for w in wls]
    caches = [synth.kv_cache(w) for w in wls]
    oracles = [oracle.Oracle.for_workload(w, c, per_head=opts.get("per_head", 0), ring_bf16=opts.get("ring_bf16", 0))
               for w, c in zip(wls, caches)]
    eager = [DeviceRun(w, c, **opts) for w, c in zip(wls, caches)]
    graph = [DeviceRun(w, c, **opts) for w, c in zip(wls, caches)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for r in graph:
            mac.mac_decode_step(r.st, r.q, r.pos, r.K, r.V, None, r.lens, r.out, r.lse, r.hit, r.mpos)
    hits = 0
    for t in range(wls[0].steps):
        for l, r in enumerate(graph):
            st = streams[l]
            r.q.copy_(torch.from_numpy(np.ascontiguousarray(st.q[t])))
            r.pos.copy_(torch.from_numpy(st.rope_pos[t]))
            r.lens.copy_(torch.from_numpy(st.seq_lens[t]))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        for l in range(L):
            st, c = streams[l], caches[l]
            y = (graph[l].out.cpu().numpy(), graph[l].lse.cpu().numpy(), graph[l].hit.cpu().numpy(),
                 graph[l].mpos.cpu().numpy())
            ref = oracles[l].step(st.q[t], st.rope_pos[t], c.K, c.V, c.block_table, st.seq_lens[t])
            np.testing.assert_array_equal(y[2], ref.hit, err_msg="hit mask, layer %d step %d" % (l, t))
            np.testing.assert_array_equal(y[3], ref.match_pos, err_msg="match position, layer %d step %d" % (l, t))
            assert float(np.abs(y[0] - ref.out).max()) <= OUT_TOL, "out, layer %d step %d" % (l, t)
            assert float(np.abs(y[1] - ref.lse).max()) <= LSE_TOL, "lse, layer %d step %d" % (l, t)
            x = eager[l].step(st.q[t], st.rope_pos[t], st.seq_lens[t])
            for u, v in zip(x, y):
                np.testing.assert_array_equal(u, v, err_msg="graph vs eager, layer %d step %d" % (l, t))
            hits += int(ref.hit.sum())
    assert hits > 0
    assert all(r.st.get_status() == 0 for r in graph)


@pytest.mark.parametrize("tune", [
    {"whole_unit_keys": 0},                                           # every range cut over CTAs
    {"whole_unit_keys": 0, "piece_cost": 0, "min_keys_per_cta": 16},  # many tiny pieces per unit
    {"whole_unit_keys": 1 << 20},                                     # every unit done by one CTA
    {"piece_cost": 1 << 16, "min_keys_per_cta": 1},                   # one piece per CTA at most
])
def test_work_split_settings_keep_parity(tune):
    """How the keys are divided among CTAs changes only rounding, never decisions."""
    wl = synth.WORKLOADS["paged_mixed"].with_(B=4, L0=(9000, 1500, 300, 4100), steps=12)
    compare_stream(wl, synth.queries(wl), synth.kv_cache(wl), tune=tune)


def test_bounded_wait_times_out_and_context_stays_usable():
    """A wait that nothing satisfies gives up after its limit: the status word
    says MAC_DEV_TIMEOUT, the launch ends on its own, and the next steps on the
    same context match the oracle."""
    import time
    import kv_cache_reuse_b200 as mac
    torch, dev = torch_dev()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    t0 = time.time()
    mac.mac_selftest_wait_timeout(status)
    torch.cuda.synchronize()
    dt = time.time() - t0
    assert int(status.item()) == mac.MAC_DEV_TIMEOUT
    assert 1.5 < dt < 30.0
    wl = synth.WORKLOADS["tiny"].with_(steps=8)
    r = compare_stream(wl, synth.queries(wl), synth.kv_cache(wl))
    assert r["hits"] > 0


def test_nan_query_misses_and_stays_local():
    wl = synth.WORKLOADS["llama8b_32k"].with_(B=2, L0=(700, 900), steps=6)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    gpu = DeviceRun(wl, cache)
    for t in range(wl.steps):
        q = stream.q[t].copy()
        if t == 4:
            q[1, 5, 3] = np.nan  # KV head 1 of sequence 1
        out, lse, hit, mpos = gpu.step(q, stream.rope_pos[t], stream.seq_lens[t])
        if t == 4:
            assert hit[1, 1] == 0 and mpos[1, 1] == -1  # a NaN distance never matches
            assert np.isnan(out[1, 5]).all() and np.isnan(lse[1, 5])  # only the poisoned head
            ok = np.ones(out.shape[:2], bool)
            ok[1, 5] = False
            assert np.isfinite(out[ok]).all() and np.isfinite(lse[ok]).all()
    assert gpu.st.get_status() == 0


def test_bad_page_and_seq_len_flagged():
    import kv_cache_reuse_b200 as mac
    wl = synth.WORKLOADS["paged_mixed"].with_(B=3, L0=(100, 200, 300), steps=3)
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    bt = cache.block_table.copy()
    bt[1, 2] = cache.num_pages + 5  # sequence 1 reads its page 2 at every step
    bad = synth.KVCache(cache.K, cache.V, bt, cache.max_seq, cache.num_pages)
    gpu = DeviceRun(wl, bad)
    out, lse, hit, mpos = gpu.step(stream.q[0], stream.rope_pos[0], stream.seq_lens[0])
    assert np.isnan(out[1]).all() and np.isnan(lse[1]).all()
    assert np.isfinite(out[0]).all() and np.isfinite(out[2]).all()
    assert gpu.st.get_status() == mac.MAC_DEV_BAD_PAGE
    lens = stream.seq_lens[1].copy()
    lens[2] = bad.max_seq + 1
    out, lse, hit, mpos = gpu.step(stream.q[1], stream.rope_pos[1], lens)
    assert np.isnan(out[2]).all()
    st = gpu.st.get_status()
    assert st & mac.MAC_DEV_BAD_SEQ_LEN and st & mac.MAC_DEV_BAD_PAGE
    assert gpu.st.get_status() == 0  # cleared by the read
