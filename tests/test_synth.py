"""The seeded input generators against their published definitions (CPU)."""
import numpy as np

from workloads import synth


def test_splitmix64_reference_outputs():
    # SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) from state 0: its first three outputs
    assert [int(x) for x in synth.u64(0, 3)] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_stream_offsets_are_slices():
    whole = synth.u64(12345, 50)
    assert np.array_equal(synth.u64(12345, 20, offset=30), whole[30:])


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -20, -2.0, 0.0])
    # 1 + 2^-8 is halfway between bf16 1.0 (0x3F80) and 1.0078125 (0x3F81): ties go to even
    assert [int(b) for b in synth.f64_to_bf16_bits(x)] == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xC000, 0x0000]


def test_normals_have_unit_moments():
    z = synth.normal_f64(synth.stream_seed(7, 1), 1 << 20)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1.0) < 5e-3
