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
