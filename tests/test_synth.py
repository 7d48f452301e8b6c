"""The seeded input generator that both the CUDA path and the oracle draw from
(kv_cache_attention_states_b200/synth.py): reproducible per-tensor streams,
round-to-nearest-even storage conversion, and workloads whose shapes,
positions and chunking are the five configurations' (8 query heads, one KV
head, head_dim 256)."""
import numpy as np
import torch

from kv_cache_attention_states_b200 import synth


def test_streams_are_reproducible_and_independent_of_draw_order():
    a1 = synth.draw(3, "k", (7, 256), "f32")
    b1 = synth.draw(3, "v", (7, 256), "f32")
    b2 = synth.draw(3, "v", (7, 256), "f32")
    a2 = synth.draw(3, "k", (7, 256), "f32")
    assert np.array_equal(a1, a2) and np.array_equal(b1, b2)
    assert not np.array_equal(a1, b1)
    assert not np.array_equal(a1, synth.draw(4, "k", (7, 256), "f32"))


def test_normal_draws_have_the_requested_scale():
    x = synth.normal(0, "q", (4096, 256), std=0.5).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 0.5) < 0.01
    assert np.array_equal(synth.normal(0, "q", (8, 4), std=0.5),
                          synth.normal(0, "q", (8, 4)) * np.float32(0.5))


def _bf16_rne_bits(x: np.ndarray) -> np.ndarray:
    # round to nearest even on the bit pattern: add 0x7fff plus the lowest
    # kept bit, drop the low 16 bits (finite inputs)
    b = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def test_storage_rounding_is_round_to_nearest_even():
    x = synth.normal(1, "r", (100000,), std=3.0)
    # ties and near-ties around bf16 and f16 spacing
    x = np.concatenate([x, np.float32([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -11,
                                       1.0 + 3 * 2.0 ** -11, -2.5, 65504.0, 1e-7])])
    bf = synth.to_storage(x, "bf16")
    assert bf.dtype == np.uint16
    assert np.array_equal(bf, _bf16_rne_bits(x))
    assert np.array_equal(bf, torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    h = synth.to_storage(x, "f16")
    assert np.array_equal(h, x.astype(np.float16))
    # ties go to even: 1 + 2^-8 lies halfway between bf16 neighbours 1 and 1 + 2^-7
    assert _bf16_rne_bits(np.float32([1.0 + 2.0 ** -8]))[0] == np.float32(1.0).view(np.uint32) >> 16
    t = synth.as_torch(bf, "bf16")
    assert t.dtype == torch.bfloat16 and np.array_equal(t.view(torch.int16).numpy().view(np.uint16), bf)


def test_tiny_f32_workload():
    w = synth.tiny_f32()
    assert (w.q_dtype, w.kv_dtype, w.capacity) == ("f32", "f32", 320)
    assert w.prefill == [(256, 48)]                                # positions 256-303
    assert [c[0] - 1 for c in w.decode_ctx] == list(range(304, 320))  # queries at 304-319


def test_decode_f16_workloads():
    for length in (256, 4096, 16384):
        w = synth.decode_f16(length)
        assert (w.q_dtype, w.kv_dtype) == ("f32", "f16")
        assert [c[0] for c in w.decode_ctx] == list(range(length, length + 64))
        assert w.capacity == length + 64


def test_prefill_16k_workload():
    w = synth.prefill_bf16_16k()
    assert (w.q_dtype, w.kv_dtype, w.std) == ("bf16", "bf16", 0.5)
    assert w.prefill == [(768 * i, 768) for i in range(21)] + [(16128, 256)]
    assert sum(r for _, r in w.prefill) == 16384


def test_window_workload():
    w = synth.window_bf16()
    assert w.window == 512 and w.kv_dtype == "bf16"
    assert w.prefill == [(768 * i, 768) for i in range(5)] + [(3840, 256)]
    assert [c[0] - 1 for c in w.decode_ctx] == list(range(4096, 4160))


def test_ragged_workload():
    w = synth.ragged_f16(0)
    assert (w.batch, w.kv_dtype, w.q_dtype, w.capacity) == (8, "f16", "f32", 131072)
    assert len(w.decode_ctx) == 32
    start = np.array(w.decode_ctx[0])
    assert ((start >= 1024) & (start + 31 <= 131072)).all()
    for t, c in enumerate(w.decode_ctx):
        assert list(np.array(c) - start) == [t] * 8
    assert np.array_equal(start, synth.ragged_f16(0).decode_ctx[0])
    assert not np.array_equal(start, synth.ragged_f16(1).decode_ctx[0])


def test_long_chunk_workload():
    w = synth.long_chunk_bf16()
    assert w.prefill == [(130304, 768)] and w.capacity == 131072
