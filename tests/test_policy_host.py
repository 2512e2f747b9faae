"""The mixed-precision policy search (weight_quantised_gemm_b200.policy) on
the host: its cosine algebra against the cosine computed directly, its
dynamic programme against brute force, and an end-to-end run on outputs the
oracle computes at 4 and 8 bits."""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle as O
import weight_quantised_gemm_b200.policy as P
import workloads as WL


def _random_layers(g, L, sizes=(3, 5, 8), correlated=True):
    """L layers with dense outputs of different lengths and 4/8-bit outputs
    with noise of different strength (partly along d, so <e, d> != 0)."""
    dense, quant, nbytes = [], [], []
    for l in range(L):
        n = int(g.choice(sizes)) * 16
        d = g.standard_normal(n) * g.uniform(0.5, 2.0)
        q = {}
        for bits, amp in ((4, 0.12), (8, 0.008)):
            e = g.standard_normal(n) * amp * g.uniform(0.5, 2.0)
            if correlated:
                e += g.uniform(-0.05, 0.05) * amp * d
            q[bits] = d + e
        dense.append(d)
        quant.append(q)
        nbytes.append({4: n * 9 // 2, 8: n * 17 // 2})
    layers = [P.layer_stats(f"l{i}", dense[i], quant[i], nbytes[i]) for i in range(L)]
    return layers, dense, quant


def _direct_cosine(dense, quant, choice):
    d = np.concatenate(dense)
    q = np.concatenate([quant[i][b] for i, b in enumerate(choice)])
    return float(q @ d / math.sqrt((q @ q) * (d @ d)))


def test_cosine_from_per_layer_terms_is_the_direct_cosine():
    g = np.random.default_rng(1)
    layers, dense, quant = _random_layers(g, 5)
    for choice in itertools.product((4, 8), repeat=5):
        a = {f"l{i}": b for i, b in enumerate(choice)}
        assert P.cosine(layers, a) == pytest.approx(_direct_cosine(dense, quant, choice), rel=1e-13, abs=1e-15)


def test_layer_stats_takes_torch_tensors_and_checks_shapes():
    d = torch.arange(8, dtype=torch.float32)
    st = P.layer_stats("x", d, {4: d + 1}, {4: 10})
    assert st.dense_energy == float((d.double() ** 2).sum())
    assert st.options[4].err == 8.0 and st.options[4].cross == float(d.double().sum())
    with pytest.raises(ValueError):
        P.layer_stats("x", d, {4: d[:4]}, {4: 10})


def _stats_layers(g, L, options=(4, 8), with_cross=False):
    layers = []
    for i in range(L):
        size = int(g.choice([1000, 2500, 4000]))
        opts = {}
        for j, b in enumerate(sorted(options)):
            err = float(g.uniform(0.5, 2.0)) * 10.0 ** (-j)
            opts[b] = P.Option(b, size * b // 4 + 7 * i, float(g.uniform(-0.1, 0.1)) * err if with_cross else 0.0, err)
        layers.append(P.LayerStats(f"l{i}", 1000.0, opts))
    return layers


def _key(front):
    return [(p.nbytes, round(p.err, 9), tuple(sorted(p.bits.items()))) for p in front]


@pytest.mark.parametrize("seed,options", [(2, (4, 8)), (3, (2, 4, 8)), (4, (1, 4, 8))])
def test_dynamic_programme_matches_brute_force(seed, options):
    """With no cross term the cosine is monotone in the error energy, so the
    exact programme's front (resolution 1) equals the enumerated one."""
    g = np.random.default_rng(seed)
    layers = _stats_layers(g, 7, options)
    brute = P.frontier(layers)                                   # 7 <= 16: enumerated
    dp = P.frontier(layers, exhaustive_max=0, resolution_bytes=1)
    assert _key(dp) == _key(brute)
    assert brute[0].nbytes == sum(min(o.nbytes for o in l.options.values()) for l in layers)
    assert brute[-1].err == pytest.approx(sum(min(o.err for o in l.options.values()) for l in layers))


def test_bucketed_programme_stays_within_its_resolution():
    g = np.random.default_rng(5)
    layers = _stats_layers(g, 9, (4, 8))
    exact = P.frontier(layers, exhaustive_max=0, resolution_bytes=1)
    r = 500
    coarse = P.frontier(layers, exhaustive_max=0, resolution_bytes=r)
    assert len(coarse) <= len(exact)
    for p in exact:   # every exact point has a coarse one at most 9 buckets larger and no less accurate
        assert any(c.nbytes <= p.nbytes + 9 * r and c.err <= p.err * (1 + 1e-12) for c in coarse)


def test_cheapest_and_most_accurate_match_enumeration_with_cross_terms():
    g = np.random.default_rng(6)
    layers, dense, quant = _random_layers(g, 6)
    allp = []
    for choice in itertools.product((4, 8), repeat=6):
        a = {f"l{i}": b for i, b in enumerate(choice)}
        allp.append((sum(l.options[a[l.name]].nbytes for l in layers), _direct_cosine(dense, quant, choice), a))
    cos_all4 = [c for n, c, a in allp if set(a.values()) == {4}][0]
    cos_all8 = [c for n, c, a in allp if set(a.values()) == {8}][0]
    for target in np.linspace(cos_all4, cos_all8, 7):
        want = min((n for n, c, _ in allp if c >= target - 1e-12), default=None)
        got = P.cheapest(layers, target - 1e-12)
        assert got is not None and got.nbytes == want
    for budget in sorted({n for n, _, _ in allp})[::5]:
        want = max(c for n, c, _ in allp if n <= budget)
        assert P.most_accurate(layers, budget).cosine == pytest.approx(want, rel=1e-12)
    assert P.cheapest(layers, 1.5) is None
    assert P.most_accurate(layers, 0) is None


def test_policy_on_oracle_outputs_orders_4_and_8_bits():
    """End to end on quantised outputs the oracle computes: three linears of a
    block, each at 4 and 8 bits, against dense fp64. All-4 is the smallest
    point of the front and all-8 the most accurate; 8-bit error is far below
    4-bit error for every layer."""
    shapes = [(64, 256, 512), (64, 512, 256), (64, 128, 512)]
    layers = []
    for i, (M, N, K) in enumerate(shapes):
        X, W, _ = WL.random_case(40 + i, M, N, K, 4, with_bias=False)
        dense = O.bf16_bits_to_f64(X) @ W.astype(np.float64).T
        outs, sizes = {}, {}
        for bits in (4, 8):
            p, s, b = O.pack_ref(W, bits, 64)
            outs[bits] = O.qgemm_ref(X, p, s, b, bits, 64, K, None)
            sizes[bits] = p.nbytes + s.nbytes + b.nbytes
        st = P.layer_stats(f"lin{i}", dense, outs, sizes)
        assert st.options[8].err < st.options[4].err / 100
        layers.append(st)
    front = P.frontier(layers)
    assert set(front[0].bits.values()) == {4} and set(front[-1].bits.values()) == {8}
    assert all(a.nbytes < b.nbytes and a.cosine < b.cosine for a, b in zip(front, front[1:]))
    assert 0.99 < front[0].cosine < front[-1].cosine < 1.0
