"""The seeded input recipe (synth.py): deterministic per seed, the layouts
the library takes, and planted needles and mixtures built as the workload
definitions state (a needle query is 4 k_j + N(0, 1) with j before the
window; a mixture is 2 (k_j1 + ... + k_j4) + N(0, 1))."""

import torch

from hierarchical_sparse_attention_recsa_b200 import synth

TINY = synth.WORKLOADS["tiny-4k"]


def test_kv_is_seeded_and_laid_out_head_major():
    K1, V1, r1 = synth.make_kv(TINY, 300, seed=3, batch=2)
    K2, V2, r2 = synth.make_kv(TINY, 300, seed=3, batch=2)
    K3, _, _ = synth.make_kv(TINY, 300, seed=4, batch=2)
    assert K1.shape == V1.shape == (2, TINY.n_kv_heads, 300, TINY.head_dim)
    assert K1.dtype == TINY.dtype and r1.dtype == torch.float32 and r1.shape == (TINY.head_dim,)
    assert torch.equal(K1, K2) and torch.equal(V1, V2) and torch.equal(r1, r2)
    assert not torch.equal(K1, K3)
    # r ~ N(0, 1/d): its squared norm is about 1
    assert 0.5 < float((r1 ** 2).sum()) < 2.0


def test_model_shaped_kv_has_a_per_channel_scale():
    w = synth.Workload("scaled", 4096, 128, 4, 2, 64, 16, 8, 512, torch.float32, True)
    K, V, _ = synth.make_kv(w, 4096, seed=5, batch=1)
    sd = K[0].std(dim=1)                      # [H_kv, d]: one scale per (head, channel)
    # LogNormal(0, 0.5) channel scales: spread well beyond the sampling noise
    # of a unit-variance channel over 4096 rows
    assert float(sd.max() / sd.min()) > 2.0
    assert 0.6 < float(sd.log().std()) / 0.5 < 1.4


def test_needles_point_at_an_earlier_key_outside_the_window():
    L = 2000
    K, _, _ = synth.make_kv(TINY, L, seed=6, batch=1)
    pos = torch.full((1, 64), L - 1, dtype=torch.int64)
    Q, kind, npos = synth.make_queries(TINY, K, pos, seed=7, n_needles=16)
    assert int((kind == 1).sum()) == 16 and int((kind == 2).sum()) == 0
    G = TINY.n_q_heads // TINY.n_kv_heads
    for i in torch.nonzero(kind[0] == 1).flatten().tolist():
        j = int(npos[0, i])
        assert 0 <= j < L - TINY.window
        for h in range(TINY.n_q_heads):
            k = K[0, h // G, j].float()
            resid = Q[0, i, h].float() - 4.0 * k     # the N(0, 1) part
            assert abs(float(resid.std()) - 1.0) < 0.35
            assert float(torch.nn.functional.cosine_similarity(Q[0, i, h].float(), k,
                                                              dim=0)) > 0.9


def test_mixture_fraction_and_needle_fraction():
    w = synth.Workload("mix", 4096, 64, 2, 1, 16, 16, 4, 64, torch.float32, False,
                       needle_frac=0.1, mixture_frac=0.2)
    K, _, _ = synth.make_kv(w, 4096, seed=8, batch=1)
    pos = torch.full((1, 4000), 4095, dtype=torch.int64)
    _, kind, _ = synth.make_queries(w, K, pos, seed=9)
    frac1 = float((kind == 1).float().mean())
    frac2 = float((kind == 2).float().mean())
    assert abs(frac1 - 0.1) < 0.02 and abs(frac2 - 0.2) < 0.03
