"""The seeded input generator: determinism, shapes and bf16 rounding (checked against torch's cast)."""
import numpy as np
import torch

import poetx_inputs as I


def test_bf16_rounding_matches_torch_cast():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 3,
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -0.0, 65504.0], np.float32)])
    ours = I.round_to_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
    bits = I.bf16_bits(ours)
    assert np.array_equal((bits.astype(np.uint32) << 16).view(np.float32), ours)


def test_layer_draw_is_deterministic_and_shaped():
    s = I.small_shape(64, 32, 16, 3, 10, dtype="bf16")
    a, b = I.make_layer(s, 5), I.make_layer(s, 5)
    for f in ("pi_L", "pi_R", "theta_R", "theta_P", "W0", "X", "dY"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    assert a.theta_R.shape == (2, 120) and a.theta_P.shape == (4, 120)
    assert sorted(a.pi_L.tolist()) == list(range(32)) and sorted(a.pi_R.tolist()) == list(range(64))
    assert a.X.shape == (10, 64) and a.dY.shape == (10, 32) and a.W0.shape == (32, 64)
    assert np.array_equal(I.round_to_bf16(a.W0), a.W0)


def test_workload_table():
    w = I.WORKLOADS["llama8b_attn_4096_b256_bf16"]
    assert (w.d_in, w.d_out, w.b, w.k, w.n_tokens, w.nb_in) == (4096, 4096, 256, 3, 2048, 16)
    assert I.WORKLOADS["layer256_b32_f32"].nb_out == 8


def test_stack_layers_and_theta_only_draws():
    L8 = I.stack_layers("llama8b_stack_32x7_b256_bf16")
    L13 = I.stack_layers("llama13b_stack_40x7_b512_bf16_mem")
    assert len(L8) == 224 and len(L13) == 280
    assert [seed for _, _, seed in L8[:2]] == [1400, 1401] and L8[-1][2] == 1623
    assert [seed for _, _, seed in L13[:2]] == [1500, 1501] and L13[-1][2] == 1779
    assert sum(s.nb_in + s.nb_out for _, s, _ in L8) == 32 * (32 + 20 + 20 + 32 + 72 + 72 + 72)
    # make_theta reproduces make_layer's theta draws exactly
    _, sh, seed = L13[6]
    tR, tP = I.make_theta(sh, seed)
    full = I.make_layer(sh, seed, n_tokens=2, with_activations=False)
    assert np.array_equal(tR, full.theta_R) and np.array_equal(tP, full.theta_P)
