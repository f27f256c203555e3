"""The seeded input generators follow their stated recipe (CPU, reduced sizes).

Recipe: K, V ~ N(0, 1) per channel; q_h = tau_h g_h; per (sequence, kv-head) round(1% of N)
heavy tokens K = 3 sqrt(128) q_h*/|q_h*| + xi aimed at one q-head h* of the group; sinks at
positions 0-3, K = 2 sqrt(128) u + xi with u the normalised mean of the group's unit queries;
pages either identity blocks or one random permutation of the pool.  Pruner rows: probability
vectors (fp64 sum one, rounded to fp32), half Gaussian-logit rows, half Zipf rank profiles, a
share with exact ties.
"""
import numpy as np

from workloads import synth

D = 128


def _row(wl, b, kvh, pos):
    return wl.k[wl.page_table[b, pos // 16], kvh, pos % 16].astype(np.float64)


def test_decode_workload_layout_and_determinism():
    a = synth.make_decode("t", 2, 8, 2, [100, 37], seed=3, permute_pages=True)
    b = synth.make_decode("t", 2, 8, 2, [100, 37], seed=3, permute_pages=True)
    c = synth.make_decode("t", 2, 8, 2, [100, 37], seed=4, permute_pages=True)
    assert a.q.dtype == np.float16 and a.k.dtype == np.float16 and a.v.dtype == np.float16
    assert a.q.shape == (2, 8, D) and a.k.shape == (7 + 3, 2, 16, D) == a.v.shape
    assert a.page_table.dtype == np.int32 and a.page_table.shape == (2, 7)
    # one permutation of the pool dealt in order; -1 past each sequence
    used = np.concatenate([a.page_table[0, :7], a.page_table[1, :3]])
    assert sorted(used.tolist()) == list(range(10))
    assert np.all(a.page_table[1, 3:] == -1)
    for f in ("q", "k", "v", "page_table"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
    assert not np.array_equal(a.k, c.k)


def test_heavy_tokens_and_sinks_follow_the_recipe():
    n, hq, hkv = 2000, 8, 2
    wl = synth.make_decode("t", 1, hq, hkv, [n], seed=11)
    g = hq // hkv
    heavy = wl.extra["heavy"]
    for kvh in range(hkv):
        mine = [h for h in heavy if h[1] == kvh]
        assert len(mine) == round(0.01 * n)
        for _, _, pos, owner in mine:
            assert 4 <= pos < n and kvh * g <= owner < (kvh + 1) * g
            k = _row(wl, 0, kvh, pos)
            u = wl.q[0, owner].astype(np.float64)
            u /= np.linalg.norm(u)
            # 3 sqrt(D) along the owner's unit query, plus unit-variance noise
            assert abs(k @ u - 3 * np.sqrt(D)) < 5.0
            assert np.linalg.norm(k - (k @ u) * u) < 1.5 * np.sqrt(D)
        units = [wl.q[0, h].astype(np.float64) / np.linalg.norm(wl.q[0, h].astype(np.float64))
                 for h in range(kvh * g, (kvh + 1) * g)]
        s = np.mean(units, axis=0)
        s /= np.linalg.norm(s)
        for pos in range(4):
            assert abs(_row(wl, 0, kvh, pos) @ s - 2 * np.sqrt(D)) < 5.0
    # ordinary tokens: unit-variance channels, no drift toward the queries
    heavy_pos = {(h[1], h[2]) for h in heavy}
    plain = np.stack([_row(wl, 0, 0, p) for p in range(4, n) if (0, p) not in heavy_pos])
    assert abs(plain.mean()) < 0.02 and abs(plain.std() - 1.0) < 0.02


def test_pruner_rows_follow_the_recipe():
    w, info = synth.config5_rows(200, 1024, seed=2, tie_frac=0.05)
    assert w.dtype == np.float32 and w.shape == (200, 1024)
    assert np.all(w > 0)
    assert np.all(np.abs(w.astype(np.float64).sum(axis=1) - 1.0) < 1e-5)
    fam = info["family"]
    assert 60 < int((fam == 0).sum()) < 140            # about half each
    assert int(info["ties"].sum()) == 10
    for r in np.nonzero(info["ties"])[0]:
        assert np.unique(w[r]).size < 1024              # exact ties present
    for r in np.nonzero(fam == 1)[0]:
        if not info["ties"][r]:
            # Zipf: the sorted row is r^-s up to the normalisation
            srt = np.sort(w[r].astype(np.float64))[::-1]
            s = info["param"][r]
            ratio = srt[:8] / srt[0]
            assert np.allclose(ratio, np.arange(1, 9) ** (-s), rtol=1e-5)
    again, _ = synth.config5_rows(200, 1024, seed=2, tie_frac=0.05)
    assert np.array_equal(w, again)


def test_temperature_recipe_divides_the_query():
    # q_h = g_h / tau_h: tau_h * q_h has unit-variance channels whatever tau_h is
    wl = synth.make_decode("t", 2, 16, 4, [64, 64], seed=5, temperature=True)
    taus = wl.extra["tau"]
    assert taus.min() >= 0.25 and taus.max() <= 8.0
    g = wl.q.astype(np.float64) * taus[:, :, None]
    assert abs(g.std() - 1.0) < 0.05 and abs(g.mean()) < 0.05
    plain = synth.make_decode("t", 2, 16, 4, [64, 64], seed=5)
    # the same draws g_h as the scaled recipe (q_h = tau_h g_h), up to fp16 rounding
    assert np.allclose(plain.q.astype(np.float64) / taus[:, :, None], g, rtol=2e-3, atol=2e-3)


def test_multi_head_layers_mix_focused_and_diffuse_heads():
    """With tau as a logit temperature the 32K layer's heads span focused and diffuse regimes
    (oracle kept fractions on an 8K-context copy of the layer, same seed); the diffuse variant
    keeps most candidates in every head."""
    from oracle import twl_oracle as O
    from tests.twl_checks import group_workload

    def kept_fractions(wl):
        out = []
        for kvh in range(wl.num_kv_heads):
            r = O.decode_step(group_workload(wl, 0, kvh), with_attention=False)
            out += [d["kept"].size / d["cand"].size for d in r["heads"].values()]
        return np.array(out)

    fr = kept_fractions(synth.config2(n=8192))
    assert np.median(fr) < 0.02 and fr.max() > 0.2, fr
    fd = kept_fractions(synth.config_diffuse(n=8192))
    assert fd.min() > 0.5, fd
