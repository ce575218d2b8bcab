"""The seeded input generator: deterministic, shaped as each workload states,
and bf16 rounding identical to torch's round-to-nearest-even conversion."""
import numpy as np
import torch

from self_sparse_speculative_b200 import workloads as W


def test_bf16_rounding_matches_torch_bit_exact():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -1e-30], np.float32)])
    # exact halfway points between bf16 neighbours, both parities
    base = rng.integers(0, 0x7F70, 1000).astype(np.uint32) << 16      # finite values only
    halves = (base | 0x8000).view(np.float32)
    x = np.concatenate([x, halves])
    ours = W.round_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = W.bf16_bits_to_float32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_workload_shapes_and_determinism():
    for idx in (0, 1, 2):
        wl = W.Workload(W.spec(idx), seed=0)
        s = wl.spec
        assert wl.q_draft.shape == (s.gamma, s.num_seqs, s.num_q_heads, s.head_dim)
        assert wl.q_verify.shape == (s.num_seqs, s.rows, s.num_q_heads, s.head_dim)
        assert wl.block_table.shape == (s.num_seqs, wl.max_pages_per_seq)
        used = np.concatenate([wl.block_table[b, :n] for b, n in enumerate(wl.pages_per_seq)])
        assert np.array_equal(np.sort(used), np.arange(wl.num_pages_total))
        if s.context:
            assert np.all(wl.context_lens == s.context)
        else:
            assert np.all(wl.context_lens % s.page_size == 0)
            assert wl.context_lens.min() >= s.ragged_lo - s.page_size and wl.context_lens.max() <= s.ragged_hi
        wl2 = W.Workload(W.spec(idx), seed=0)
        assert np.array_equal(wl.kv_pages("K", [0, 3]), wl2.kv_pages("K", [0, 3]))
        assert not np.array_equal(wl.kv_pages("K", [0]), wl.kv_pages("V", [0]))
    t, d = W.Workload(W.spec(1)).logits_for_seq(0)
    assert t.shape == (5, 151936) and d.shape == (4, 151936) and t.dtype == np.uint16
    tf, df = W.to_float64(t, "bf16"), W.to_float64(d, "bf16")
    assert 1.9 < tf.std() < 2.1 and 0.45 < (df - tf[:4]).std() < 0.55


def test_outlier_channels_present():
    wl = W.Workload(W.spec(1), seed=0)
    k = W.to_float64(wl.kv_pages("K", range(8)), "bf16")      # [8, H, P, D]
    var = k.var(axis=(0, 2))                                      # [H, D]
    for h in range(8):
        ch = wl._outlier["K"][0][h]
        assert var[h, ch].mean() > 1.2 * np.delete(var[h], ch).mean()
