"""The seeded input generators shared by the tests, the bench and the smoke check (CPU).

They hold none of the method's arithmetic; both sides of every parity test read their inputs from
them, so their determinism and recipe are what these tests pin: the same seed gives the same
tensors, the draw order is fixed (optional tensors never change the others), the gate follows
f = lb + (1 - lb) sigmoid(x), and packed sequences are slices of one token stream.
"""
import numpy as np
import torch

from linear_attention_hgrn2_b200 import inputs as I


def test_same_seed_same_tensors_and_fixed_draw_order():
    a = I.make_inputs(2, 9, 3, 4, 5, torch.float32, 0.5, seed=11)
    b = I.make_inputs(2, 9, 3, 4, 5, torch.float32, 0.5, seed=11, with_dO=True, h0_sigma=0.1, dhT_sigma=0.2)
    c = I.make_inputs(2, 9, 3, 4, 5, torch.float32, 0.5, seed=12)
    for k in ("q", "i", "log_f"):
        assert torch.equal(a[k], b[k]), k          # optional draws come after, never before
        assert not torch.equal(a[k], c[k]), k      # another seed, other values
    assert set(b) == {"q", "i", "log_f", "dO", "h0", "dhT"}
    assert b["h0"].shape == (2, 3, 4, 5) and b["h0"].dtype == torch.float32
    assert abs(float(b["h0"].std()) - 0.1) < 0.05 and abs(float(b["dhT"].std()) - 0.2) < 0.1


def test_gate_follows_the_lower_bounded_sigmoid():
    x = np.linspace(-30.0, 30.0, 601)
    for lb in (0.0, 0.5, 0.95):
        lf = I.gate_log_f(x, lb)
        f = lb + (1.0 - lb) / (1.0 + np.exp(-x))
        np.testing.assert_allclose(lf, np.log(f), rtol=1e-12, atol=1e-15)   # f ~ 1: absolute rounding
        assert np.all(lf <= 0.0) and np.all(np.diff(lf) > 0.0)     # a decay, increasing in x
        if lb > 0:
            assert np.all(lf >= np.log(lb))
    # lb = 0 stays finite and accurate far in the tail, where log(sigmoid) ~ x
    assert I.gate_log_f(np.array([-800.0]), 0.0)[0] == -800.0


def test_bf16_inputs_are_the_rounded_draws():
    a = I.make_inputs(1, 5, 2, 8, 8, torch.float32, 0.9, seed=3)
    b = I.make_inputs(1, 5, 2, 8, 8, torch.bfloat16, 0.9, seed=3)
    for k in ("q", "i", "log_f"):
        assert b[k].dtype == torch.bfloat16
        assert torch.equal(a[k].to(torch.bfloat16), b[k]), k


def test_document_lengths_fill_the_total_exactly():
    for seed in range(5):
        lens = I.document_lengths(16384, 512, seed=seed)
        assert sum(lens) == 16384 and min(lens) >= 1
        assert lens == I.document_lengths(16384, 512, seed=seed)
    assert all(n >= 4 for n in I.document_lengths(1000, 50, seed=1, min_len=4)[:-1])


def test_packed_sequences_are_slices_of_one_stream():
    lens = [3, 1, 7, 5]
    p = I.make_varlen(lens, 2, 4, 6, torch.float32, 0.5, seed=21, h0_sigma=0.1, with_dO=True)
    cu = p["cu_seqlens"].tolist()
    assert cu == [0, 3, 4, 11, 16] and p["cu_seqlens"].dtype == torch.int32
    whole = I.make_inputs(1, 16, 2, 4, 6, torch.float32, 0.5, seed=21, with_dO=True)
    for k in ("q", "log_f", "i", "dO"):
        assert torch.equal(p[k], whole[k][0]), k
    assert p["h0"].shape == (4, 2, 4, 6)


def test_scalar_decay_inputs():
    s = I.make_scalar_inputs(2, 7, 3, 4, 5, torch.float32, 0.5, seed=5, with_dO=True, h0_sigma=0.1)
    assert s["q"].shape == (2, 7, 3, 4) and s["k"].shape == (2, 7, 3, 4) and s["v"].shape == (2, 7, 3, 5)
    assert s["log_g"].shape == (2, 7, 3) and bool((s["log_g"] <= 0).all())
    assert bool((s["log_g"] >= np.log(0.5)).all())
    assert abs(float(s["k"].std()) - 0.5) < 0.2              # k ~ N(0, 1/d_k)


def test_headline_workload_is_the_bench_configuration():
    w = I.TRAIN
    assert (w.B, w.H, w.T, w.dk, w.dv, w.dtype, w.lb) == (8, 16, 2048, 128, 128, torch.bfloat16, 0.95)
    assert w.name == "train_fwdbwd_bf16_B8_H16_T2048_d128"
    assert (I.TRAIN_D64.H * I.TRAIN_D64.dk, I.TRAIN_D256.H * I.TRAIN_D256.dk) == (2048, 2048)
