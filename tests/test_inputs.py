"""The seeded input stream: the torch evaluation (used for full-size device inputs) draws
the same numbers as the numpy definition.  On the CPU the two agree bit for bit."""
import numpy as np

from swin3d_window_attention_b200 import inputs


def test_torch_stream_matches_numpy_stream_on_cpu():
    for ti, sigma in ((0, 1.0), (7, 0.7), (123, 0.1)):
        a = inputs.normal_f32(300_001, tensor_index=ti, sigma=sigma)
        b = inputs.normal_f32_torch(300_001, "cpu", tensor_index=ti, sigma=sigma, chunk_pairs=1 << 16).numpy()
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
        ab = inputs.f32_to_bf16_bits(a)
        bb = inputs.torch_bf16_to_bits(inputs.normal_bf16_torch((300_001,), "cpu", tensor_index=ti, sigma=sigma))
        assert np.array_equal(ab, bb)


def test_stream_statistics():
    x = inputs.normal_f32(1 << 20, tensor_index=3).astype(np.float64)
    assert abs(x.mean()) < 5e-3 and abs(x.std() - 1.0) < 5e-3
