"""The seeded generators: determinism, shapes, distributions and the token tree."""
import numpy as np

from speech_encoder_attention_b200 import inputs


def test_encoder_inputs_are_deterministic_and_shaped():
    spec = inputs.ENCODER_WORKLOADS["tiny"]
    a = inputs.make_encoder_inputs(spec)
    b = inputs.make_encoder_inputs(spec)
    assert a.x.shape == (64, 128) and a.w_qkv.shape == (384, 128)
    assert a.b_q.shape == (128,) and a.b_v.shape == (128,)
    assert a.x.dtype == np.float16
    for f in ("x", "w_qkv", "b_q", "b_v"):
        np.testing.assert_array_equal(getattr(a, f), getattr(b, f))


def test_batch_override_keeps_leading_windows():
    spec = inputs.ENCODER_WORKLOADS["windows8"]
    small = inputs.make_encoder_inputs(spec, batch=2)
    assert small.x.shape == (3000, 1280)
    full = inputs.make_encoder_inputs(spec)
    np.testing.assert_array_equal(full.x[:3000], small.x)
    np.testing.assert_array_equal(full.w_qkv, small.w_qkv)


def test_window_offsets_differ_per_window():
    full = inputs.make_encoder_inputs(inputs.ENCODER_WORKLOADS["windows8"])
    means = full.x.astype(np.float64).reshape(8, 1500, 1280).mean(axis=(1, 2))
    assert np.all(np.abs(means) < 0.55)
    assert np.ptp(means) > 0.1


def test_distributions():
    full = inputs.make_encoder_inputs(inputs.ENCODER_WORKLOADS["window"])
    assert abs(full.x.astype(np.float64).std() - 1.0) < 0.01
    assert abs(full.w_qkv.astype(np.float64).std() - 0.02) < 0.001
    assert abs(full.b_q.astype(np.float64).std() - 0.01) < 0.002


def test_chunk_workload_is_eleven_full_chunks_and_a_short_one():
    spec = inputs.ENCODER_WORKLOADS["chunks"]
    assert spec.t == 11 * 200 + 125 and spec.chunk_len == 200


def test_token_tree_shape_and_counts():
    spec = inputs.VERIFY_WORKLOADS["verify"]
    inp = inputs.make_verify_inputs(spec)
    assert spec.t_q == 80 and spec.slots == 448
    assert inp.bits.shape == (80, 14) and inp.bits.dtype == np.uint32
    allowed = inputs.unpack_bits(inp.bits, 448)
    counts = allowed.sum(axis=1)
    # prompt (8) + one slot per beam step (72) + position in the block (1..16)
    np.testing.assert_array_equal(counts, np.tile(np.arange(81, 97), 5))
    assert counts.sum() == 7080
    # every row admits itself and the whole prompt, and nothing after itself
    for r, s in enumerate(inp.query_slot):
        assert allowed[r, s]
        assert allowed[r, :8].all()
        assert not allowed[r, s + 1:].any()
    # beams do not see each other's blocks
    for b in range(5):
        rows = slice(16 * b, 16 * b + 16)
        for b2 in range(5):
            if b2 != b:
                assert not allowed[rows, 368 + 16 * b2: 368 + 16 * b2 + 16].any()


def test_token_tree_parents_are_earlier_slots():
    spec = inputs.VERIFY_WORKLOADS["verify"]
    inp = inputs.make_verify_inputs(spec)
    p = inp.parent
    assert p[0] == -1
    assert np.all(p[1:] < np.arange(1, len(p)))
    assert np.all(p[1:] >= 0)


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(0)
    a = rng.random((7, 70)) < 0.5
    np.testing.assert_array_equal(inputs.unpack_bits(inputs.pack_bits(a), 70), a)
    bits = inputs.pack_bits(a)
    assert bits.shape == (7, 3)
    # bits past the last slot stay clear
    assert np.all(bits[:, 2] >> np.uint32(6) == 0)


def test_varlen_lengths_are_seeded_and_in_range():
    spec = inputs.ENCODER_WORKLOADS["varlen8"]
    a, b = inputs.encoder_lengths(spec), inputs.encoder_lengths(spec)
    np.testing.assert_array_equal(a, b)
    assert a.dtype == np.int32 and a.shape == (spec.batch,)
    assert a.min() >= 500 and a.max() <= spec.t
    assert inputs.encoder_lengths(inputs.ENCODER_WORKLOADS["windows8"]) is None


def test_drafter_inputs_shapes_and_determinism():
    spec = inputs.DRAFTER_WORKLOADS["drafter_causal"]
    a, b = inputs.make_drafter_inputs(spec), inputs.make_drafter_inputs(spec)
    assert a.q.shape == (spec.beams * spec.t_q, spec.d_model)
    assert a.k.shape == a.v.shape == (spec.beams * spec.t_kv, spec.d_model)
    assert a.sinks.shape == (spec.n_heads,) and a.sinks.dtype == np.float32
    np.testing.assert_array_equal(a.k, b.k)
    assert spec.t_kv == spec.context + spec.block


def test_bench_pair_counts_match_brute_force():
    """The bench's algorithmic flop counts: allowed pairs counted in closed form
    against an element-by-element count of the allowed matrix."""
    import bench
    import oracle
    for t, w in [(10, 1), (10, 3), (37, 8), (1500, 256)]:
        assert bench.band_pairs(t, w) == int(oracle.allowed_range(t, t, window=w).sum())
    spec = inputs.ENCODER_WORKLOADS["varlen8"]
    lens = inputs.encoder_lengths(spec)
    assert bench.encoder_pairs(spec) == sum(int(oracle.allowed_range(spec.t, spec.t, q_len=int(n),
                                                                       kv_len=int(n)).sum()) for n in lens)
    assert bench.encoder_valid_rows(spec) == int(lens.sum())


def test_q8_inputs_layout_and_determinism():
    spec = inputs.Q8_WORKLOADS["q8_tiny"]
    a, b = inputs.make_q8_inputs(spec), inputs.make_q8_inputs(spec)
    np.testing.assert_array_equal(a.w_blocks, b.w_blocks)
    d = spec.d_model
    assert a.w_blocks.shape == (3 * d, d // 32 * 34) and a.w_blocks.dtype == np.uint8
    # the packed bytes carry exactly the drawn scales and values
    blk = a.w_blocks.reshape(3 * d, d // 32, 34)
    np.testing.assert_array_equal(blk[:, :, :2].copy().view("<f2")[..., 0], a.scales)
    np.testing.assert_array_equal(blk[:, :, 2:].copy().view(np.int8).reshape(3 * d, d), a.qs)
    assert a.qs.min() >= -127 and a.qs.max() <= 127


def test_kernel_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    """Stored ncu counters stay valid across comment edits, not code edits."""
    import bench
    src = tmp_path / "k.cuh"
    src.write_text("// header\nint f(int x) {  // trailing\n  return x + 1; /* note */\n}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ["k.cuh"])
    h0 = bench.kernel_source_hash()
    src.write_text("// a different header\n/* block\n comment */\nint f(int x) {\n  return x + 1;\n}\n")
    assert bench.kernel_source_hash() == h0
    src.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.kernel_source_hash() != h0


def test_clock_sampler_with_a_fake_nvml(monkeypatch):
    """The bench's clock sampler, against a fake NVML module: it samples while
    its region runs and reports the median clock of the samples taken under
    load and the union of their reasons (idle dropped)."""
    import sys
    import threading
    import time
    import types

    import bench
    seq = iter([(1965, 100, 0x4), (1900, 0, 0x8), (1950, 90, 0x0), (1965, 80, 0x1)] * 10000)
    lock = threading.Lock()
    cur = {}

    def clock(h, which):
        with lock:
            cur["s"] = next(seq)
            return cur["s"][0]

    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0, nvmlInit=lambda: None, nvmlDeviceGetHandleByIndex=lambda i: object(),
        nvmlDeviceGetMaxClockInfo=lambda h, w: 1965, nvmlDeviceGetClockInfo=clock,
        nvmlDeviceGetUtilizationRates=lambda h: types.SimpleNamespace(gpu=cur["s"][1]),
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: cur["s"][2])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    sampler = bench.ClockSampler(0)
    with sampler:
        time.sleep(0.05)
    rec = sampler.summary()
    assert rec["samples"] >= 4 and 0 < rec["samples_under_load"] < rec["samples"]
    assert rec["sm_max_mhz"] == 1965 and rec["sm_mhz"] in (1950, 1965)
    # the sample with no load (its hw_slowdown bit included) is left out
    assert rec["reasons"] == ["sw_power_cap"]
