"""The seeded input generators (CPU only)."""

import numpy as np
import torch

from oracle import doc_layout, rope_angles_f64
from workloads import CONFIGS, config_by_name, make_workload, rope_tables_f32, round_to_bf16


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * s for s in (1e-3, 1.0, 1e3)])
    # exact ties: values halfway between two bf16 neighbours
    ties = (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(round_to_bf16(x), want)


def test_rope_tables_are_the_oracle_angles_rounded_once_to_f32():
    for T, D in ((128, 64), (512, 128)):
        c32, s32 = rope_tables_f32(T, D, 10000.0)
        c64, s64 = rope_angles_f64(T, D, 10000.0)
        assert c32.dtype == np.float32 and c32.shape == (T, D // 2)
        assert np.array_equal(c32, c64.astype(np.float32))
        assert np.array_equal(s32, s64.astype(np.float32))


def test_packed_documents_fill_rows_within_the_length_range():
    cfg = config_by_name("packed_docs")
    w = make_workload(cfg)
    cu = w.cu_seqlens
    assert cu[0] == 0 and cu[-1] == cfg.B * cfg.T
    lens = np.diff(cu)
    assert np.all(lens > 0) and np.all(lens <= cfg.doc_max)
    for r in range(cfg.B + 1):
        assert r * cfg.T in cu
    # only a row's last document may be shorter than doc_min (truncated)
    ends = set(r * cfg.T for r in range(1, cfg.B + 1))
    for e, n in zip(cu[1:], lens):
        if e not in ends:
            assert n >= cfg.doc_min
    doc_layout(cfg.B, cfg.T, cu)   # the oracle accepts it


def test_workloads_are_seeded_and_bf16_representable():
    cfg = config_by_name("gpt12m_layer")
    a = make_workload(cfg, B=2, T=64)
    b = make_workload(cfg, B=2, T=64)
    for x, y in ((a.q, b.q), (a.do, b.do)):
        assert np.array_equal(x, y)
    assert np.array_equal(round_to_bf16(a.q), a.q)
    assert abs(float(a.do.std()) - 0.01) < 1e-3
    peaky = make_workload(config_by_name("decoder237m_layer"), B=1, H=2, T=256)
    assert abs(float(peaky.q.std()) - 1.5) < 0.02


def test_config_table():
    assert [c.name for c in CONFIGS] == ["tiny_fp32", "gpt12m_layer", "decoder237m_layer",
                                         "long_context_8k", "packed_docs"]
    c = config_by_name("long_context_8k")
    assert c.nominal_flops == 7 * 1 * 16 * 8192 * 8192 * 128


def test_projection_workloads_are_seeded_shaped_and_bf16():
    from workloads import PROJ_CONFIGS, make_proj_workload, proj_config_by_name

    for cfg in PROJ_CONFIGS:
        w = make_proj_workload(cfg, B=1, T=256)
        c = w.cfg
        F = (c.H + 2 * c.H_kv) * c.D
        assert w.x.shape == (1, 256, c.C) and w.w_qkv.shape == (F, c.C)
        assert w.w_o.shape == (c.C, c.H * c.D) and w.o.shape == (1, c.H, 256, c.D)
        assert w.dq.shape == (1, c.H, 256, c.D) and w.dk.shape == w.dv.shape == (1, c.H_kv, 256, c.D)
        assert w.dy.shape == (1, 256, c.C)
        for a in (w.x, w.w_qkv, w.w_o, w.o, w.dq, w.dk, w.dv, w.dy):
            assert a.dtype == np.float32 and np.array_equal(round_to_bf16(a), a)
        # fan-in scale of the weights, 0.01 for the output gradients
        assert abs(w.w_qkv.std() * np.sqrt(c.C) - 1.0) < 0.05
        assert abs(w.dy.std() / 0.01 - 1.0) < 0.05
        if c.packed:
            cu = w.cu_seqlens
            assert cu[0] == 0 and cu[-1] == 256 and np.all(np.diff(cu) > 0)
            assert np.all(np.diff(cu)[:-1] <= c.doc_hi)
    a = make_proj_workload(proj_config_by_name("proj_small_d64"))
    b = make_proj_workload(proj_config_by_name("proj_small_d64"))
    assert np.array_equal(a.x, b.x) and np.array_equal(a.cu_seqlens, b.cu_seqlens)
    c = make_proj_workload(proj_config_by_name("proj_small_d64"), seed=99)
    assert not np.array_equal(a.x, c.x)
