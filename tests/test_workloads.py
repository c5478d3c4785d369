"""The seeded input generators: deterministic, row-addressable, and shaped as stated."""

import numpy as np
import torch

from sparse_attention_token_02_b200 import workloads as W


def test_rows_are_addressable_and_deterministic():
    full = W.normal_rows(3, 1, 0, 9000, 8)
    part = W.normal_rows(3, 1, 4000, 8500, 8)
    assert np.array_equal(full[4000:8500], part)
    assert np.array_equal(full, W.normal_rows(3, 1, 0, 9000, 8))
    assert not np.array_equal(full, W.normal_rows(4, 1, 0, 9000, 8))


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * np.float32(3.0)
    ours = W.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_workload_shapes_and_pairs():
    c1 = W.tiny()
    assert (c1.H, c1.d, c1.top_k, c1.seq_lens, c1.seed) == (4, 64, 32, (512,), 0)
    assert c1.pairs == 512 * 513 // 2 == 131328
    c2 = W.decode()
    assert c2.pairs == 32 * 32768 and c2.kind == "decode"
    c3 = W.prefill()
    assert c3.pairs == 16384 * 16385 // 2 == 134225920
    c4 = W.prefill8()
    assert c4.pairs == 65536 * 65537 // 2 == 2147516416
    c5 = W.decode8()
    assert len(c5.seq_lens) == 16 and all(4096 <= L <= 131072 for L in c5.seq_lens)
    assert c5.pairs == sum(2 * L - 1 for L in c5.seq_lens)


def test_inputs_distribution_and_outliers():
    wl = W.scaled(W.prefill(), seq_lens=(2000,), q_lens=(2000,))
    k = W.key_rows(wl, 0)
    norms = np.linalg.norm(k, axis=1)
    big = norms > 2.5 * np.sqrt(wl.d)
    assert big.sum() == 20                       # 1% of the rows, x4
    w = W.weight_rows(wl, 0, 100)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6) and np.all(w > 0)
    inp = W.make_inputs(W.scaled(W.decode(), seq_lens=(300, 300), q_lens=(1, 1)))
    assert inp["q_bits"].shape == (2, 64, 128) and inp["k_bits"][0].shape == (300, 128)
