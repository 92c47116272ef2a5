"""The seeded input generator: bf16 rounding, reproducibility, recipes."""
import numpy as np
import torch

from selective_state_space_36_b200 import inputs as I


def test_bf16_rounding_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        # exact ties between two bf16 values, both parities
                        (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
                        np.array([0.0, -0.0, 1e-40, -3.0e38, 65504.0], dtype=np.float32)])
    ours = I.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = I.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_slices_reproduce_full_draw():
    cfg = I.ScanConfig("t", 2, 3 * I.CHUNK_ROWS + 17, 24, 16, io="bf16", seed=9)
    full = I.draw_tensor(cfg, "u")
    for t0, t1 in [(0, 5), (I.CHUNK_ROWS - 3, I.CHUNK_ROWS + 4), (2 * I.CHUNK_ROWS + 1, cfg.seqlen)]:
        assert np.array_equal(I.draw_tensor(cfg, "u", t0, t1), full[:, t0:t1])
    assert np.array_equal(I.draw_tensor(cfg, "B", threads=1), I.draw_tensor(cfg, "B", threads=4))
    # different tensors and batch rows are different streams
    assert not np.array_equal(full[0], full[1])
    assert not np.array_equal(I.draw_tensor(cfg, "z"), full)


def test_recipes():
    A, D, bias = I.channel_params(2, 4096, 16, "uniform")
    assert np.array_equal(A[7], -(np.arange(16, dtype=np.float32) + 1))
    dt0 = np.logaddexp(0.0, bias.astype(np.float64))
    assert dt0.min() >= 1e-3 * (1 - 1e-5) and dt0.max() <= 1e-1 * (1 + 1e-5)
    assert 0.5 <= D.min() and D.max() <= 1.5
    _, D1, _ = I.channel_params(0, 64, 16, "one")
    assert np.all(D1 == 1.0)
    cfg = I.TINY_F32
    x = I.scan_inputs(cfg)
    assert x["u"].dtype == np.float32 and x["u"].shape == (1, 256, 64)
    assert x["B"].shape == (1, 256, 16)
    dl = x["delta"].astype(np.float64)
    assert abs(dl.std() - 0.5) < 0.02 and abs(x["u"].std() - 1.0) < 0.02
    dec = I.DecodeConfig("d", 4, 40, 16, steps=3, seed=4)
    st = I.decode_step_inputs(dec, 1)
    dt = I.bf16_bits_to_f32(st["dt"])
    assert dt.shape == (4, 40) and np.all(dt > 0)
    assert not np.array_equal(st["x"], I.decode_step_inputs(dec, 2)["x"])
