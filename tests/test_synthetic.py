"""Checks of the seeded generator and of the workload sizes against the pages."""
import numpy as np

from synthetic import gen, workloads as W


def test_streams_are_deterministic_and_independent():
    a = gen.activations(W.DECODE_35B, 3, 7, 4)
    b = gen.activations(W.DECODE_35B, 3, 7, 4)
    c = gen.activations(W.DECODE_35B, 3, 8, 4)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    # a (layer, step) stream can be regenerated alone, and a prefix is a prefix
    assert np.array_equal(gen.activations(W.DECODE_35B, 3, 7, 2), a[:2])


def test_normals_moments():
    z = gen.normals(gen.stream_key(1, 2, 3, 4), 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01


def test_bf16_rounding_is_nearest_even():
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -20], np.float32)
    out = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(f))
    assert out.tolist() == [1.0, 1.0, 1.0 + 4 * 2 ** -8, -2.5, 1.0 + 2 ** -7]


def test_expert_pool_size_matches_pages():
    """The 284B model's MXFP4 expert pool is about 140 GB on the pages
    (post.smzdm.com/p/a825qpgl, section 一); 40 layers x 256 experts of
    [2048x4096]x2 + [4096x2048] MXFP4 tensors in 4096-aligned blocks give 136.9 GB."""
    w = W.DECODE_284B
    total = w.L * w.E * W.expert_block_bytes(w)
    assert W.expert_block_bytes(w) == 13369344 == 3264 * 4096
    assert abs(total / 1e9 - 140) / 140 < 0.03
    assert W.expert_block_bytes(W.DECODE_35B) == 2654208 == 648 * 4096


def test_slot_counts():
    assert W.n_slots(W.DECODE_35B) == 1536
    assert W.n_slots(W.DECODE_284B) == 2570
    assert [W.n_slots(W.stress_variant(1.0, p)) for p in W.STRESS_POOL] == [1024, 2560, 5120]
    assert W.n_slots(W.TINY) == 16 and W.n_slots(W.PREFILL_35B) == 128


def test_weight_recipes():
    t = gen.expert_weights(W.TINY, 0, 3)
    c, s, ts = t["gate"]
    assert c.shape == (256, 128) and s.shape == (256, 8) and ts == 1.0
    assert s.min() >= 123 and s.max() <= 127
    n = gen.expert_weights(W.Workload(name="n", H=256, I=64, E=2, k=1, L=1, fmt=W.NVFP4, seed=1,
                                      batches=(1,), steps=1, zipf_s=0, weight_recipe="normal"),
                           0, 1)
    c, s, ts = n["down"]
    assert c.shape == (256, 32) and s.shape == (256, 4) and ts > 0
