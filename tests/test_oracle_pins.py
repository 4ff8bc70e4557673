"""Pins of the fp64 oracle against facts it does not define itself.

Each test fixes one part of the oracle with something independent of its
code: a textbook formula written differently (complex RoPE, plain softmax),
a closed form worked by hand (tests/golden), brute force on tiny inputs, or
an invariant that a plausible mistake would break.  Source of the method:
MAC-Attention, page 1 (abstract).
"""
import numpy as np
import pytest

import oracle
import synth
from tests.dense_ref import (dense_attention, dense_step, decode, load_hand_example, rope_complex)


def _tiny(**kw):
    return synth.WORKLOADS["tiny"].with_(**kw)


# ---------------------------------------------------------------- RoPE pins
def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(11)
    for D in (64, 128):
        for pos in (0, 1, 7, 1023, 131199):
            q = rng.standard_normal(D).astype(np.float32)
            got = oracle.rope(q, pos, 5e5)
            # the fp64 angle pos * theta^(-2i/D) carries ~1e-16 * pos radians of rounding
            tol = 1e-13 + 1e-15 * pos * float(np.abs(q).max())
            np.testing.assert_allclose(got, rope_complex(q, pos, 5e5), rtol=0, atol=tol)


def test_rope_is_identity_at_zero_and_relative():
    rng = np.random.default_rng(12)
    D = 128
    q = rng.standard_normal(D).astype(np.float32)
    k = rng.standard_normal(D).astype(np.float32)
    np.testing.assert_array_equal(oracle.rope(q, 0, 1e4), q.astype(np.float64))
    # norm preserved; score depends only on the position difference
    for m, n in ((5, 2), (1000, 17), (70000, 69000)):
        qm = oracle.rope(q, m, 1e4)
        kn = oracle.rope(k, n, 1e4)
        assert abs(np.linalg.norm(qm) - np.linalg.norm(q.astype(np.float64))) < 1e-12
        rel = oracle.rope(q, m - n, 1e4)
        assert abs(qm @ kn - rel @ k.astype(np.float64)) < 1e-9


# --------------------------------------------------------- partial / merge
def _rand_kv(rng, L, D):
    K = synth.f32_to_bf16_bits(rng.standard_normal((L, D)).astype(np.float32))
    V = synth.f32_to_bf16_bits(rng.standard_normal((L, D)).astype(np.float32))
    return K, V


def test_partial_equals_dense_softmax():
    rng = np.random.default_rng(13)
    L, D = 300, 64
    K, V = _rand_kv(rng, L, D)
    q = rng.standard_normal(D)
    o, m, l = oracle.partial(q, K, V, 0, L)
    o_ref, lse_ref = dense_attention(q[None], decode(K), decode(V))
    np.testing.assert_allclose(o, o_ref[0], rtol=0, atol=1e-13)
    assert abs(m + np.log(l) - lse_ref[0]) < 1e-12
    o, m, l = oracle.partial(q, K, V, 5, 5)
    assert m == -np.inf and l == 0.0 and not o.any()


@pytest.mark.parametrize("scale", [1.0, 1e3])
def test_merge_of_any_partition_equals_dense(scale):
    """Stable merge (page 1, complete stage): any partition, any order, equals dense."""
    rng = np.random.default_rng(14)
    L, D = 257, 64
    K, V = _rand_kv(rng, L, D)
    q = rng.standard_normal(D) * scale  # scale 1e3 gives logits of order +-1e4
    o_ref, lse_ref = dense_attention(q[None], decode(K), decode(V))
    for trial in range(20):
        ncut = rng.integers(0, 12)
        cuts = np.sort(rng.integers(0, L + 1, size=ncut))
        edges = np.concatenate([[0], cuts, [L]])  # repeated cuts give empty parts
        parts = [oracle.partial(q, K, V, int(a), int(b)) for a, b in zip(edges[:-1], edges[1:])]
        rng.shuffle(parts)
        acc = parts[0]
        for p in parts[1:]:
            acc = oracle.merge(acc, p)
        o, m, l = acc
        np.testing.assert_allclose(o, o_ref[0], rtol=0, atol=1e-11)
        assert abs((m + np.log(l)) - lse_ref[0]) <= 1e-12 * max(1.0, abs(lse_ref[0]))


def test_merge_empty_is_identity():
    D = 8
    o = np.arange(D, dtype=np.float64)
    e = (np.zeros(D), -np.inf, 0.0)
    r = oracle.merge(e, (o, 1.5, 2.0))
    assert r[1] == 1.5 and r[2] == 2.0 and np.array_equal(r[0], o)
    r = oracle.merge(e, e)
    assert r[1] == -np.inf and r[2] == 0.0 and not r[0].any()


# ------------------------------------------------------------ worked example
def test_hand_worked_example():
    g, K, V, qs = load_hand_example()
    sh = g["shape"]
    orc = oracle.Oracle(sh["B"], sh["Hq"], sh["Hkv"], sh["D"], sh["W"], sh["band"], sh["tau"],
                        sh["rope_theta"], 0, sh["max_seq"], 0)
    for st, q in zip(g["steps"], qs):
        r = orc.step(q, np.array([st["rope_pos"]], np.int32), K, V, None, np.array([st["seq_len"]], np.int32))
        assert int(r.hit[0, 0]) == st["hit"]
        assert int(r.match_pos[0, 0]) == st["match_pos"]
        np.testing.assert_allclose(r.out[0, :, 0], st["out0"], atol=1e-6)
        np.testing.assert_allclose(r.out[0, :, 1], st["out1"], atol=1e-6)
        np.testing.assert_allclose(r.out[0, :, 2:], 0.0, atol=0)
        np.testing.assert_allclose(r.lse[0], st["lse"], atol=1e-6)
        if "dense_out0" in st:  # the reuse really differs from dense here
            assert abs(st["out0"] - st["dense_out0"]) > 0.4


# ----------------------------------------------------------- whole-step pins
def _run(wl, steps=None, stream=None, cache=None, tau=None, band=None, rope_zero=False, cut_mode=0):
    stream = stream or synth.queries(wl, steps)
    cache = cache or synth.kv_cache(wl, steps)
    orc = oracle.Oracle.for_workload(wl, cache, tau=tau, band=band, cut_mode=cut_mode)
    res = []
    for t in range(stream.q.shape[0]):
        rp = np.zeros_like(stream.rope_pos[t]) if rope_zero else stream.rope_pos[t]
        res.append(orc.step(stream.q[t], rp, cache.K, cache.V, cache.block_table, stream.seq_lens[t]))
    return stream, cache, res


@pytest.mark.parametrize("G", [1, 4, 16])
def test_distance_equal_to_threshold_is_a_miss(G):
    """The match test is strict: an entry at distance exactly tau misses, and
    one ulp more of tau makes it a hit.  The queries are multiples of 1/8 and
    differ by 0.5 in one element per head, so the mean over heads of the
    squared L2 distance is exactly 0.25 in any precision."""
    wl = _tiny(Hq=G, Hkv=1, steps=3)
    cache = synth.kv_cache(wl)
    stream = synth.queries(wl)
    q0 = ((np.arange(G * wl.D).reshape(1, G, wl.D) % 16 - 8) / 8).astype(np.float32)
    q1 = q0.copy()
    q1[0, :, 3] += np.float32(0.5)
    for tau, hit in ((0.25, False), (np.nextafter(0.25, 1.0), True)):
        orc = oracle.Oracle.for_workload(wl, cache, tau=tau)
        orc.step(q0, stream.rope_pos[0], cache.K, cache.V, cache.block_table, stream.seq_lens[0])
        r = orc.step(q1, stream.rope_pos[1], cache.K, cache.V, cache.block_table, stream.seq_lens[1])
        assert bool(r.hit[0, 0]) is hit
        assert r.d_best[0, 0] == 0.25
        if hit:
            assert r.match_pos[0, 0] == stream.seq_lens[0][0] - 1  # the first step's position


def test_equal_distances_pick_the_most_recent_entry():
    """Two window entries at the same distance: the match is the more recent
    one (its reused prefix is longer and its tail shorter)."""
    wl = _tiny(steps=5)
    cache = synth.kv_cache(wl)
    stream = synth.queries(wl)
    q = stream.q[0].copy()
    far = (q + np.float32(3.0)).astype(np.float32)
    orc = oracle.Oracle.for_workload(wl, cache, tau=1.0)
    seq = [q, far, q, q]  # steps 0 and 2 hold the same query; step 3 repeats it
    for t, qt in enumerate(seq):
        r = orc.step(qt, stream.rope_pos[t], cache.K, cache.V, cache.block_table, stream.seq_lens[t])
    assert r.hit[0, 0] and r.d_best[0, 0] == 0.0 and r.d_second[0, 0] == 0.0
    assert r.match_pos[0, 0] == stream.seq_lens[2][0] - 1


@pytest.mark.parametrize("cut_mode", [0, 1])
def test_forced_miss_equals_dense(cut_mode):
    """Threshold 0 (strict test) makes every step a miss, i.e. dense attention,
    wherever the prefix/tail cut falls."""
    wl = _tiny(steps=12)
    stream, cache, res = _run(wl, tau=0.0, cut_mode=cut_mode)
    for t, r in enumerate(res):
        assert not r.hit.any()
        o, l = dense_step(wl, cache, stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        np.testing.assert_allclose(r.out, o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.lse, l, rtol=0, atol=1e-12)


def test_forced_miss_paged_equals_dense():
    wl = synth.WORKLOADS["paged_mixed"].with_(B=3, Hq=8, Hkv=2, D=64, L0=(100, 37, 250), steps=6,
                                              W=4, band=8, tau=0.0)
    stream, cache, res = _run(wl)
    for t, r in enumerate(res):
        o, l = dense_step(wl, cache, stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        np.testing.assert_allclose(r.out, o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.lse, l, rtol=0, atol=1e-12)


def test_exact_repeats_without_rotation_equal_dense():
    """Identity RoPE and exact repeats: the reused state is the current query's own."""
    wl = _tiny(steps=24, sigma=0.0)
    stream = synth.queries(wl, sigma=0.0)
    stream, cache, res = _run(wl, stream=stream, rope_zero=True)
    nhit = 0
    for t, r in enumerate(res):
        nhit += int(r.hit.sum())
        o, l = dense_step(wl, cache, stream.q[t], np.zeros(wl.B, np.int32), stream.seq_lens[t])
        np.testing.assert_allclose(r.out, o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.lse, l, rtol=0, atol=1e-12)
    assert nhit >= 6


@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (6, 2), (8, 1), (32, 2), (32, 1), (64, 1)])
def test_group_sizes_forced_miss_equals_dense(Hq, Hkv):
    """Groups of 1 (multi-head), 3, 8, 16, 32 and 64 (multi-query) query heads
    per KV head: a forced miss is dense attention of every query head over its
    KV head."""
    wl = _tiny(steps=8, Hq=Hq, Hkv=Hkv)
    stream, cache, res = _run(wl, tau=0.0)
    for t, r in enumerate(res):
        assert r.out.shape == (wl.B, Hq, wl.D) and r.hit.shape == (wl.B, Hkv)
        o, l = dense_step(wl, cache, stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        np.testing.assert_allclose(r.out, o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.lse, l, rtol=0, atol=1e-12)


@pytest.mark.parametrize("Hq,Hkv", [(3, 3), (10, 2), (8, 1), (16, 1), (64, 1)])
def test_group_sizes_band_covering_hits_equal_dense(Hq, Hkv):
    """With the band covering the context, hits reuse an empty prefix: the
    stored and reused states of every head in the group must come out exact."""
    wl = _tiny(L0=(40,), steps=16, band=200, Hq=Hq, Hkv=Hkv)
    stream, cache, res = _run(wl)
    nhit = 0
    for t, r in enumerate(res):
        nhit += int(r.hit.sum())
        o, l = dense_step(wl, cache, stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        np.testing.assert_allclose(r.out, o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.lse, l, rtol=0, atol=1e-12)
    assert nhit >= 4


@pytest.mark.parametrize("cut_mode", [0, 1])
def test_band_covering_context_equals_dense(cut_mode):
    """band >= p_t + 1 puts every reuse boundary at 0: hits are exact under any RoPE."""
    wl = _tiny(L0=(40,), steps=16, band=200)
    stream, cache, res = _run(wl, cut_mode=cut_mode)
    nhit = 0
    for t, r in enumerate(res):
        nhit += int(r.hit.sum())
        o, l = dense_step(wl, cache, stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        np.testing.assert_allclose(r.out, o, rtol=0, atol=1e-12)
    assert nhit >= 4


def test_hits_differ_from_dense_and_stay_convex():
    """A real reuse is an approximation; its output stays a convex mix of V rows."""
    wl = _tiny(steps=32)
    stream, cache, res = _run(wl)
    Vd = decode(cache.V[0, :, 0])
    diff = 0.0
    for t, r in enumerate(res):
        L = int(stream.seq_lens[t][0])
        lo, hi = Vd[:L].min(axis=0), Vd[:L].max(axis=0)
        assert np.all(r.out[0] >= lo - 1e-12) and np.all(r.out[0] <= hi + 1e-12)
        assert np.all(np.isfinite(r.lse))
        if r.hit.any():
            o, _ = dense_step(wl, cache, stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
            diff = max(diff, float(np.abs(r.out - o).max()))
    assert diff > 1e-6


@pytest.mark.parametrize("cut_mode", [0, 1])
def test_hit_cost_is_constant_in_context_length(cut_mode):
    """On a hit the keys attended are b + (p_t - p_s) + 1 whatever the context (page 1);
    one fewer when the band ends at the match position itself (cut_mode 1)."""
    per_L = {}
    for L0 in (256, 4096):
        wl = _tiny(L0=(L0,), steps=20)
        stream, cache, res = _run(wl, cut_mode=cut_mode)
        keys = []
        for t, r in enumerate(res):
            if r.hit[0, 0]:
                p_t = int(stream.seq_lens[t][0]) - 1
                p_s = int(r.match_pos[0, 0])
                assert r.keys_read == wl.band + (p_t - p_s) + 1 - cut_mode
                keys.append(r.keys_read)
            else:
                assert r.keys_read == int(stream.seq_lens[t][0])
        per_L[L0] = keys
    assert per_L[256] == per_L[4096] and len(per_L[256]) > 3


@pytest.mark.parametrize("cut_mode", [0, 1])
def test_stored_prefix_is_dense_attention_up_to_the_cut(cut_mode):
    """After a miss the stored state is exact attention of the step's rotated
    query over keys [0, c), c = max(0, p - b + cut_mode), written as a plain
    softmax; an empty prefix is (o = 0, m = -inf)."""
    wl = _tiny(L0=(20,), steps=10, band=24)
    stream = synth.queries(wl)
    cache = synth.kv_cache(wl)
    orc = oracle.Oracle.for_workload(wl, cache, tau=0.0, cut_mode=cut_mode)
    K, V = decode(cache.K[0, :, 0]), decode(cache.V[0, :, 0])
    checked = empty = 0
    for t in range(wl.steps):
        orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
        p = int(stream.seq_lens[t][0]) - 1
        c = max(0, p - wl.band + cut_mode)
        q, o, m, l, pos = orc.window(0)
        assert int(pos[-1]) == p
        if c == 0:
            assert np.all(o[-1] == 0.0) and np.all(np.isneginf(m[-1]))
            empty += 1
            continue
        qr = rope_complex(stream.q[t][0].astype(np.float64), int(stream.rope_pos[t][0]), wl.rope_theta)
        o_ref, lse_ref = dense_attention(qr, K[:c], V[:c])
        np.testing.assert_allclose(o[-1], o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(m[-1] + np.log(l[-1]), lse_ref, rtol=0, atol=1e-12)
        checked += 1
    assert checked >= 4 and empty >= 1


def test_cut_mode_out_of_range_is_rejected():
    wl = _tiny(steps=2)
    with pytest.raises(ValueError):
        oracle.Oracle.for_workload(wl, synth.kv_cache(wl), cut_mode=2)


def test_warm_start_stores_prefill_queries_and_prefix_states():
    """A window seeded from n prefill positions holds each position's own query,
    its position, and exact attention of its rotated query over [0, c) (plain
    softmax), oldest first; the window is emptied first."""
    wl = _tiny(L0=(60,), steps=8, band=24)
    stream = synth.queries(wl)
    cache = synth.kv_cache(wl)
    orc = oracle.Oracle.for_workload(wl, cache)
    orc.step(stream.q[0], stream.rope_pos[0], cache.K, cache.V, None, stream.seq_lens[0])  # to be discarded
    n = 5
    orc.warm_start(stream.q[1:1 + n], stream.rope_pos[1:1 + n], cache.K, cache.V, None, stream.seq_lens[1:1 + n])
    q, o, m, l, pos = orc.window(0)
    assert len(pos) == n
    K, V = decode(cache.K[0, :, 0]), decode(cache.V[0, :, 0])
    for j in range(n):
        t = 1 + j
        p = int(stream.seq_lens[t][0]) - 1
        assert int(pos[j]) == p
        np.testing.assert_array_equal(q[j], stream.q[t][0])
        c = max(0, p - wl.band)
        qr = rope_complex(stream.q[t][0].astype(np.float64), int(stream.rope_pos[t][0]), wl.rope_theta)
        o_ref, lse_ref = dense_attention(qr, K[:c], V[:c])
        np.testing.assert_allclose(o[j], o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(m[j] + np.log(l[j]), lse_ref, rtol=0, atol=1e-12)


def test_warm_start_lets_the_first_decode_step_hit():
    """Without a seeded window the first decode step always misses; after a warm
    start an exact repeat of a prefill query (identity RoPE) hits it, and the
    output then equals dense attention."""
    wl = _tiny(L0=(80,), steps=6, sigma=0.0)
    stream = synth.queries(wl, sigma=0.0)
    cache = synth.kv_cache(wl)
    n = 4
    zero = np.zeros((n, wl.B), np.int32)
    orc = oracle.Oracle.for_workload(wl, cache)
    orc.warm_start(stream.q[:n], zero, cache.K, cache.V, None, stream.seq_lens[:n])
    t = n
    q = stream.q[1].copy()  # repeat of a seeded prefill query
    r = orc.step(q, np.zeros(wl.B, np.int32), cache.K, cache.V, None, stream.seq_lens[t])
    assert bool(r.hit[0, 0]) and int(r.match_pos[0, 0]) == int(stream.seq_lens[1][0]) - 1
    o, lse = dense_step(wl, cache, q, np.zeros(wl.B, np.int32), stream.seq_lens[t])
    np.testing.assert_allclose(r.out, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r.lse, lse, rtol=0, atol=1e-12)
    fresh = oracle.Oracle.for_workload(wl, cache)
    r0 = fresh.step(q, np.zeros(wl.B, np.int32), cache.K, cache.V, None, stream.seq_lens[t])
    assert not r0.hit.any()


# ---------------------------------------------------------------- match pins
def _brute_match(window, q, tau, G):
    """numpy brute force: mean-over-heads squared L2, argmin, ties to later, strict < tau."""
    best, arg = np.inf, -1
    for idx, (qe, pos) in enumerate(window):
        d = float(np.sum((q.astype(np.float64) - qe.astype(np.float64)) ** 2) / G)
        if np.isnan(d):
            continue
        if d < best or (d == best and arg >= 0 and pos >= window[arg][1]):
            best, arg = d, idx
    if arg >= 0 and best < tau:
        return True, window[arg][1]
    return False, -1


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (2, 2), (9, 3), (16, 2), (32, 1), (64, 2)])
def test_match_equals_brute_force(Hq, Hkv):
    rng = np.random.default_rng(15)
    B, D, W = 2, 8, 4
    G = Hq // Hkv
    orc = oracle.Oracle(B, Hq, Hkv, D, W, 2, 0.5, 1e4, 0, 1 << 10, 0)
    hist = [[[] for _ in range(Hkv)] for _ in range(B)]
    pool = []
    K = np.zeros((B, 1 << 10, Hkv, D), np.uint16)
    for t in range(40):
        q = np.empty((B, Hq, D), np.float32)
        for b in range(B):
            r = rng.random()
            if pool and r < 0.3:  # exact repeat of a recent step: forces ties on later duplicates
                q[b] = pool[int(rng.integers(0, len(pool)))][b]
            elif pool and r < 0.6:
                q[b] = pool[-1][b] + rng.normal(0, 0.1, (Hq, D)).astype(np.float32)
            else:
                q[b] = rng.standard_normal((Hq, D)).astype(np.float32)
        if t == 17:
            q[1, 0, 0] = np.nan
        pool.append(q.copy())
        pool = pool[-3:]
        lens = np.array([t + 5, 2 * t + 9], np.int32)
        r = orc.step(q, lens - 1, K, K, None, lens)
        for b in range(B):
            for kvh in range(Hkv):
                qg = q[b, kvh * G:(kvh + 1) * G]
                win = hist[b][kvh][-W:]
                want_hit, want_pos = _brute_match(win, qg, 0.5, G)
                assert bool(r.hit[b, kvh]) == want_hit, (t, b, kvh)
                assert int(r.match_pos[b, kvh]) == want_pos, (t, b, kvh)
                hist[b][kvh].append((qg.copy(), int(lens[b]) - 1))
    # the NaN query never matches
    assert True


@pytest.mark.parametrize("name,steps", [("tiny", None), ("llama8b_32k", None), ("long_128k", None),
                                        ("paged_mixed", None), ("continuous_16k", 1024)])
def test_generator_labels_recovered_with_margin(name, steps):
    """Repeats hit their source step, fresh queries miss, with >= 1% distance margins."""
    wl = synth.WORKLOADS[name]
    stream = synth.queries(wl, steps)
    orc = oracle.Oracle(wl.B, wl.Hq, wl.Hkv, wl.D, wl.W, wl.band, wl.tau, wl.rope_theta)
    for t in range(stream.q.shape[0]):
        hit, mpos, db, ds = orc.match_step(stream.q[t], stream.seq_lens[t])
        for b in range(wl.B):
            lab = stream.label[t, b]
            if lab:
                assert hit[b].all(), (t, b)
                assert (mpos[b] == stream.rope_pos[stream.src[t, b], b]).all(), (t, b)
                assert (db[b] < 0.99 * wl.tau).all()
                assert (ds[b] >= 1.01 * db[b]).all()
            else:
                assert not hit[b].any(), (t, b)
                if t > 0:
                    assert (db[b] > 1.01 * wl.tau).all()


@pytest.mark.parametrize("Hq,Hkv,name", [(32, 1, "llama8b_32k"), (64, 1, "tiny"), (16, 1, "paged_mixed")])
def test_mqa_generator_labels_recovered_with_margin(Hq, Hkv, name):
    """Multi-query shapes (16 to 64 query heads over one KV head): repeats hit
    their source step, fresh queries miss, with >= 1% distance margins."""
    wl = synth.WORKLOADS[name].with_(Hq=Hq, Hkv=Hkv, B=min(synth.WORKLOADS[name].B, 4),
                                     L0=synth.WORKLOADS[name].L0[:4])
    stream = synth.queries(wl, 96)
    orc = oracle.Oracle(wl.B, wl.Hq, wl.Hkv, wl.D, wl.W, wl.band, wl.tau, wl.rope_theta)
    for t in range(stream.q.shape[0]):
        hit, mpos, db, ds = orc.match_step(stream.q[t], stream.seq_lens[t])
        for b in range(wl.B):
            if stream.label[t, b]:
                assert hit[b].all() and (mpos[b] == stream.rope_pos[stream.src[t, b], b]).all(), (t, b)
                assert (db[b] < 0.99 * wl.tau).all() and (ds[b] >= 1.01 * db[b]).all()
            else:
                assert not hit[b].any(), (t, b)
                if t > 0:
                    assert (db[b] > 1.01 * wl.tau).all()


# ------------------------------------------------------- per-head matching pins
@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (8, 1)])
def test_per_head_match_equals_brute_force(Hq, Hkv):
    """Per-head matching: every query head takes its own nearest entry over the
    window of its own earlier queries (numpy brute force, mean over one head)."""
    rng = np.random.default_rng(16)
    B, D, W = 2, 8, 4
    G = Hq // Hkv
    orc = oracle.Oracle(B, Hq, Hkv, D, W, 2, 0.5, 1e4, 0, 1 << 10, 0, per_head=1)
    hist = [[[] for _ in range(Hq)] for _ in range(B)]
    pool = []
    K = np.zeros((B, 1 << 10, Hkv, D), np.uint16)
    nhit = 0
    for t in range(40):
        q = np.empty((B, Hq, D), np.float32)
        for b in range(B):
            for h in range(Hq):  # each head repeats or draws fresh on its own
                r = rng.random()
                if pool and r < 0.3:
                    q[b, h] = pool[int(rng.integers(0, len(pool)))][b, h]
                elif pool and r < 0.6:
                    q[b, h] = pool[-1][b, h] + rng.normal(0, 0.1, D).astype(np.float32)
                else:
                    q[b, h] = rng.standard_normal(D).astype(np.float32)
        if t == 17:
            q[1, 0, 0] = np.nan
        pool.append(q.copy())
        pool = pool[-3:]
        lens = np.array([t + 5, 2 * t + 9], np.int32)
        r = orc.step(q, lens - 1, K, K, None, lens)
        assert r.hit.shape == (B, Hq)
        for b in range(B):
            for h in range(Hq):
                want_hit, want_pos = _brute_match(hist[b][h][-W:], q[b, h:h + 1], 0.5, 1)
                assert bool(r.hit[b, h]) == want_hit, (t, b, h)
                assert int(r.match_pos[b, h]) == want_pos, (t, b, h)
                nhit += int(want_hit)
                hist[b][h].append((q[b, h:h + 1].copy(), int(lens[b]) - 1))
    # the heads of a group disagree on some steps, or the test shows nothing
    assert 0 < nhit < 40 * B * Hq


def _heads(**kw):
    return _tiny(head_labels=True, **kw)


def test_per_head_forced_miss_equals_dense():
    wl = _heads(steps=8, Hq=4, Hkv=2)
    stream = synth.queries(wl)
    cache = synth.kv_cache(wl)
    orc = oracle.Oracle.for_workload(wl, cache, tau=0.0, per_head=1)
    for t in range(wl.steps):
        r = orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
        assert not r.hit.any()
        o, l = dense_step(wl, cache, stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        np.testing.assert_allclose(r.out, o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.lse, l, rtol=0, atol=1e-12)


@pytest.mark.parametrize("cut_mode", [0, 1])
def test_per_head_band_covering_hits_equal_dense(cut_mode):
    """Band covering the context: every head's reuse boundary is 0, so each
    head's reused state must be its own exact state, whichever entry it took."""
    wl = _heads(L0=(40,), steps=16, band=200, Hq=8, Hkv=2)
    stream = synth.queries(wl)
    cache = synth.kv_cache(wl)
    orc = oracle.Oracle.for_workload(wl, cache, cut_mode=cut_mode, per_head=1)
    mixed = 0
    for t in range(wl.steps):
        r = orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
        grp = r.hit.reshape(wl.B, wl.Hkv, wl.G)
        mixed += int((grp.any(-1) & ~grp.all(-1)).sum())
        o, l = dense_step(wl, cache, stream.q[t], stream.rope_pos[t], stream.seq_lens[t])
        np.testing.assert_allclose(r.out, o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.lse, l, rtol=0, atol=1e-12)
    assert mixed >= 4  # groups whose heads disagreed


def test_per_head_with_single_head_groups_equals_group_matching():
    """With one query head per KV head the two matching modes coincide."""
    wl = _heads(steps=24, Hq=2, Hkv=2)
    stream = synth.queries(wl)
    cache = synth.kv_cache(wl)
    a = oracle.Oracle.for_workload(wl, cache, per_head=0)
    b = oracle.Oracle.for_workload(wl, cache, per_head=1)
    for t in range(wl.steps):
        ra = a.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
        rb = b.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
        for x, y in ((ra.out, rb.out), (ra.lse, rb.lse), (ra.hit, rb.hit), (ra.match_pos, rb.match_pos)):
            np.testing.assert_array_equal(x, y)
        assert ra.keys_read == rb.keys_read


@pytest.mark.parametrize("Hq,Hkv,D", [(4, 1, 64), (32, 8, 128)])
def test_per_head_generator_labels_recovered_with_margin(Hq, Hkv, D):
    """Per-head labels: each repeated head hits its own source, fresh heads miss,
    with >= 1% margins on the threshold and between the two nearest entries."""
    base = synth.WORKLOADS["tiny"] if D == 64 else synth.WORKLOADS["llama8b_32k"]
    wl = base.with_(Hq=Hq, Hkv=Hkv, head_labels=True, steps=64)
    stream = synth.queries(wl)
    orc = oracle.Oracle(wl.B, wl.Hq, wl.Hkv, wl.D, wl.W, wl.band, wl.tau, wl.rope_theta, per_head=1)
    for t in range(wl.steps):
        hit, mpos, db, ds = orc.match_step(stream.q[t], stream.seq_lens[t])
        lab = stream.label[t]
        assert (hit.astype(bool) == lab).all(), t
        src_pos = np.where(lab, stream.rope_pos[np.maximum(stream.src[t], 0), 0], -1)
        assert (mpos == src_pos).all(), t
        assert (db[lab] < 0.99 * wl.tau).all() and (ds[lab] >= 1.01 * db[lab]).all()
        if t > 0:
            assert (db[~lab] > 1.01 * wl.tau).all()


def test_per_head_keys_read_is_the_union_of_head_ranges():
    """A KV head's keys are read once for its group: the keys attended freshly
    are p_t + 1 minus the smallest reuse boundary over its heads (0 on a miss)."""
    wl = _heads(steps=24, Hq=8, Hkv=2)
    stream = synth.queries(wl)
    cache = synth.kv_cache(wl)
    orc = oracle.Oracle.for_workload(wl, cache, per_head=1)
    for t in range(wl.steps):
        r = orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
        p_t = int(stream.seq_lens[t][0]) - 1
        want = 0
        for kvh in range(wl.Hkv):
            mp = r.match_pos[0, kvh * wl.G:(kvh + 1) * wl.G]
            first = min(max(0, int(m) - wl.band) if m >= 0 else 0 for m in mp)
            want += p_t + 1 - first
        assert r.keys_read == want, t


# ------------------------------------------------------------ bf16 ring pins
def _torch_bf16(x):
    """fp32 -> bf16 -> fp32 through torch's own conversion (round to nearest even)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def test_bf16_ring_window_holds_rounded_queries_and_states():
    """With a bf16 window every entry keeps bf16(q) and bf16(fp32(o)) of its
    prefix state (a forced-miss step's prefix state is dense attention over
    [0, c)), and m, l unrounded."""
    wl = _tiny(steps=6, L0=(300,))
    stream = synth.queries(wl)
    cache = synth.kv_cache(wl)
    orc = oracle.Oracle.for_workload(wl, cache, tau=0.0, ring_bf16=1)
    ref = oracle.Oracle.for_workload(wl, cache, tau=0.0)
    for t in range(wl.steps):
        orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
        ref.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
    q, o, m, l, pos = orc.window(0)
    rq, ro, rm, rl, rpos = ref.window(0)
    np.testing.assert_array_equal(q, _torch_bf16(stream.q[:wl.steps, 0]))
    np.testing.assert_array_equal(pos, rpos)
    np.testing.assert_array_equal(m, rm)
    np.testing.assert_array_equal(l, rl)
    # o against numpy dense attention over the stored prefix [0, c), rounded the same way
    for e in range(wl.steps):
        p = int(pos[e])
        cut = max(0, p - wl.band)
        Kd = decode(cache.K[0, :cut, 0])
        Vd = decode(cache.V[0, :cut, 0])
        qr = np.stack([rope_complex(stream.q[e, 0, h], p, wl.rope_theta) for h in range(wl.G)])
        od, _ = dense_attention(qr, Kd, Vd)
        np.testing.assert_array_equal(o[e], _torch_bf16(od.astype(np.float32)))
    assert (o != ro).any()  # the rounding is really applied


def test_bf16_ring_forced_miss_equals_dense():
    wl = _tiny(steps=8)
    stream, cache, res = _run(wl, tau=0.0)
    orc = oracle.Oracle.for_workload(wl, cache, tau=0.0, ring_bf16=1)
    for t in range(wl.steps):
        r = orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
        np.testing.assert_array_equal(r.out, res[t].out)
        np.testing.assert_array_equal(r.lse, res[t].lse)


def test_bf16_ring_first_hit_reuses_the_rounded_state():
    """The first hit of a stream (no earlier reuse, so both windows hold the
    same states up to rounding) equals the fp32-window computation with only
    the reused o replaced by bf16(o): reused state (+) amend band, (+) tail."""
    wl = _tiny(steps=40)
    stream = synth.queries(wl)
    cache = synth.kv_cache(wl)
    a = oracle.Oracle.for_workload(wl, cache)
    b = oracle.Oracle.for_workload(wl, cache, ring_bf16=1)
    K2, V2 = cache.K[0, :, 0], cache.V[0, :, 0]
    for t in range(wl.steps):
        _, wo, wm, wl_, wpos = a.window(0)  # the fp32 window before this step
        ra = a.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
        rb = b.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, None, stream.seq_lens[t])
        np.testing.assert_array_equal(ra.hit, rb.hit)
        if not ra.hit.any():
            np.testing.assert_array_equal(ra.out, rb.out)
            continue
        p_s, p_t = int(ra.match_pos[0, 0]), int(stream.seq_lens[t][0]) - 1
        e = int(np.nonzero(wpos == p_s)[0][-1])
        c_s, c_t = max(0, p_s - wl.band), max(0, p_t - wl.band)
        for h in range(wl.G):
            qr = oracle.rope(stream.q[t, 0, h], int(stream.rope_pos[t][0]), wl.rope_theta)
            reused = (_torch_bf16(wo[e, h].astype(np.float32)).astype(np.float64), wm[e, h], wl_[e, h])
            S = oracle.merge(reused, oracle.partial(qr, K2, V2, c_s, c_t))
            o, m, l = oracle.merge(S, oracle.partial(qr, K2, V2, c_t, p_t + 1))
            np.testing.assert_allclose(rb.out[0, h], o, rtol=0, atol=1e-12)
            np.testing.assert_allclose(rb.lse[0, h], m + np.log(l), rtol=0, atol=1e-12)
        assert float(np.abs(ra.out - rb.out).max()) > 0.0  # the rounding reached the output
        return
    raise AssertionError("the stream has no hit")


def test_bf16_ring_keeps_decisions_on_the_workload_margins():
    """Rounding the stored queries moves distances far less than the
    generator's margins: every decision of the stream is unchanged."""
    wl = synth.WORKLOADS["llama8b_32k"]
    stream = synth.queries(wl)
    a = oracle.Oracle(wl.B, wl.Hq, wl.Hkv, wl.D, wl.W, wl.band, wl.tau, wl.rope_theta)
    b = oracle.Oracle(wl.B, wl.Hq, wl.Hkv, wl.D, wl.W, wl.band, wl.tau, wl.rope_theta, ring_bf16=1)
    for t in range(wl.steps):
        ha, pa, _, _ = a.match_step(stream.q[t], stream.seq_lens[t])
        hb, pb, _, _ = b.match_step(stream.q[t], stream.seq_lens[t])
        np.testing.assert_array_equal(ha, hb)
        np.testing.assert_array_equal(pa, pb)
