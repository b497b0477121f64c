import numpy as np
import torch

from state_space_sequence_chunked_b200 import inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 65504.0, -3.0e38])])
    bits = inputs.bf16_bits(a)
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, ref)
    back = inputs.bf16_to_f64(bits)
    np.testing.assert_array_equal(back, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_draws_are_seeded_and_in_range():
    wl = inputs.WORKLOADS["mamba2_130m"]
    a = inputs.draw(wl, batch=1, seqlen=64)
    b = inputs.draw(wl, batch=1, seqlen=64)
    for k in ("x", "dt", "A", "B", "C", "D"):
        np.testing.assert_array_equal(a[k].bits, b[k].bits)
    assert a["h0"] is None
    dt = a["dt"].value
    assert dt.min() >= 0.99e-3 and dt.max() <= 1.01e-1
    A = a["A"].value
    assert A.max() <= -0.99 and A.min() >= -16.1
    assert a["x"].shape == (1, 64, 24, 64) and a["B"].shape == (1, 64, 1, 128)


def test_verify_draws_accepted_indices():
    wl = inputs.WORKLOADS["verify_k8"]
    d = inputs.draw(wl, batch=64)
    acc = d["accepted"]
    assert acc.dtype == np.int32 and acc.min() >= 0 and acc.max() <= 8
    assert d["h0"] is not None and d["h0"].shape == (64, 32, 128, 128)
