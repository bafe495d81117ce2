"""The seeded input recipe (CPU): determinism, SplitMix64 vector, planted keys."""
import torch

from h2o_kv_cache_b200.workload import CONFIGS, Config, gen_sequence, splitmix64, split_chunks


def test_splitmix64_published_vector():
    # first output of SplitMix64 from state 0
    assert splitmix64(0) == 0xE220A8397B1DCDAF


def test_bounds_cover_the_stream():
    for cfg in CONFIGS.values():
        b = cfg.bounds()
        assert b[0] == (0, cfg.P) and b[-1][1] == cfg.T
        assert all(b[i][1] == b[i + 1][0] for i in range(len(b) - 1))
        assert len(b) - 1 == cfg.n_chunks
    assert CONFIGS[1].n_chunks == 14 and CONFIGS[2].n_chunks == 48 and CONFIGS[3].n_chunks == 48
    assert CONFIGS[4].n_chunks == 24 and CONFIGS[0].n_chunks == 4


def test_generation_is_deterministic_and_planted():
    cfg = Config(9, "t", 1, 8, 2, 16, 64, 8, 400, 64, 32, torch.float32, 0.05)
    a = gen_sequence(cfg, 0, 0)
    b = gen_sequence(cfg, 0, 0)
    c = gen_sequence(cfg, 1, 0)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert not torch.equal(a[0], c[0])
    Q, K, V = a
    G = cfg.G
    n_plant = round(cfg.planted * cfg.T)
    for h in range(cfg.Hkv):
        u = Q[h * G:(h + 1) * G].reshape(-1, cfg.d).mean(0)
        u = u / u.norm()
        cos = (K[h] @ u) / K[h].norm(dim=1)
        assert int(((cos - 0.8).abs() < 1e-4).sum()) == n_plant


def test_split_chunks_contiguous():
    cfg = CONFIGS[0]
    Q, K, V = (x[None] for x in gen_sequence(cfg, 0, 0, T=cfg.P + 2 * cfg.S))
    ch = split_chunks(Q, K, V, [(0, cfg.P), (cfg.P, cfg.P + cfg.S)])
    assert all(t.is_contiguous() for c in ch for t in c)
    assert ch[1][0].shape == (1, cfg.Hq, cfg.S, cfg.d)
