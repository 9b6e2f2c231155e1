"""The seeded synthetic workload generator: shapes, determinism, structure."""
import math

import numpy as np
import torch

from kv_cache_top_proposal_b200 import workload


def test_configs_shapes():
    for name in workload.CONFIG_NAMES:
        c = workload.config(name)
        assert c.num_q_heads % c.num_kv_heads == 0
        assert c.kappa <= c.kappa_p
        assert c.is_proposal(0)
        assert len(c.seqlens) == c.batch
    r = workload.config("ragged16")
    assert all(4096 <= L <= 65536 for L in r.seqlens) and len(set(r.seqlens)) > 8
    assert workload.config("c128k").proposal_layers == [0, 8, 16, 24]
    assert workload.config("c8k").proposal_layers == [0, 4]


def test_generate_deterministic_and_shaped():
    cfg = workload.config("tiny")
    a = list(workload.generate(cfg, "cpu"))
    b = list(workload.generate(cfg, "cpu", layers=[2]))
    assert len(a) == 4 and len(b) == 1
    assert a[0].q.shape == (1, 4, 64) and a[0].k.shape == (1, 1024, 64)
    assert torch.equal(a[2].k, b[0].k) and torch.equal(a[2].v, b[0].v) and torch.equal(a[2].q, b[0].q)


def test_drift_and_salient_structure():
    cfg = workload.config("tiny")
    lay = list(workload.generate(cfg, "cpu"))
    sal = workload.salient_positions(cfg)[0][0]
    mask = torch.ones(1024, dtype=torch.bool)
    mask[sal] = False
    # values drift by 0.3 * N(0,1) per layer
    dv = (lay[1].v - lay[0].v).flatten()
    assert abs(dv.std().item() - 0.3) < 0.01
    dk = (lay[1].k[0, mask] - lay[0].k[0, mask]).flatten()
    assert abs(dk.std().item() - 0.3) < 0.01
    # planted keys sit at cosine 0.8 with their query head
    for l in lay:
        for i, p in enumerate(sal.tolist()):
            qh = l.q[0, i % cfg.G]
            kv = l.k[0, p]
            cos = (qh @ kv / (qh.norm() * kv.norm())).item()
            assert abs(cos - 0.8) < 1e-4


def test_rope_and_ragged_small():
    cfg = workload.config("ragged16").replace(seqlens=(37, 0, 300), batch=3, num_layers=2,
                                               num_kv_heads=2, num_q_heads=8, n_salient=4)
    lay = list(workload.generate(cfg, "cpu"))
    assert lay[0].k.shape == (2, 337, 128) and lay[0].k.dtype == torch.bfloat16
    # RoPE is a rotation: per-pair norms are preserved relative to raw keys
    cfg2 = cfg.replace(rope=False)
    raw = list(workload.generate(cfg2, "cpu"))[0]
    sal = workload.salient_positions(cfg)
    keep = torch.ones(337, dtype=torch.bool)
    for b, off in enumerate(cfg.cu_seqlens[:-1]):
        for h in range(2):
            keep[off + sal[b][h]] = False
    n1 = lay[0].k.float()[:, keep].norm(dim=-1)
    n2 = raw.k.float()[:, keep].norm(dim=-1)
    assert torch.allclose(n1, n2, rtol=2e-2)
    assert not torch.allclose(lay[0].k.float()[:, keep][:, 5:], raw.k.float()[:, keep][:, 5:])
