"""The benchmark's algorithmic accounting and its recorded-traffic guard (CPU).

The roofline fractions that ``bench.py`` reports divide algorithmic bytes or
flops by a measured time, so the counts are pinned here to the figures the
workloads fix, each added up from its parts:

* GDN prefill workload (B=4, H=16, T=4096, d=128, bf16, zero initial state):
  q, k, v read 201,326,592 B; g, beta read 2,097,152 B; o written
  67,108,864 B; states written 4,194,304 B: 274,726,912 B per call;
* dense chunked-WY flop count per head-token at d = 128, C = 64: three
  C x C x d_k products (K K^T, Q K^T, W), two C x C x d_v (U, A_qk V_new) and
  three C x d_k x d_v (W H0, Q H0, K^T V_new), 2 flop each: 180,224;
* serving decode, one state update (d = 128, bf16): fp32 state read and
  written 131,072 B, q/k/v 768 B, o 256 B, g and beta 8 B: 132,104 B;
  packed INT8 g32: codes 32,768 B, scales 4,096 B, the same 1,032 B of
  token data: 37,896 B;
* KDA prefill workload (B=2, H=32, T=8192, d=128, bf16, per-key fp32 log
  gates, zero initial state): q, k, v 402,653,184 B; g 268,435,456 B;
  beta 2,097,152 B; o 134,217,728 B; states written 4,194,304 B:
  811,597,824 B per call;
* packed varlen workload (64 sequences, H=16, d=128, bf16, scalar gate,
  random initial state read and written): 1,032 B per head-token plus
  134,217,728 B of state;
* backward on the GDN workload: 679,477,248 B (inputs read once, fp32
  gradients written once);
* the recorded DRAM traffic is reported only for the sources it was taken
  on.
"""

import bench


def test_prefill_bytes_gdn_workload():
    tok = 4 * 4096 * 16
    parts = tok * 3 * 128 * 2 + tok * 2 * 4 + tok * 128 * 2 + 4 * 16 * 128 * 128 * 4
    assert parts == 201_326_592 + 2_097_152 + 67_108_864 + 4_194_304 == 274_726_912
    got = bench.prefill_bytes(4 * 4096, 4, 16, 128, 128, 2, state_in=False, per_key=False)
    assert got == 274_726_912
    # an initial state is read as well; a per-key gate is d_k floats per token
    assert bench.prefill_bytes(4 * 4096, 4, 16, 128, 128, 2, True, False) == got + 4_194_304
    assert (bench.prefill_bytes(4 * 4096, 4, 16, 128, 128, 2, False, True)
            == got + tok * 127 * 4)


def test_prefill_bytes_kda_workload():
    tok = 2 * 8192 * 32
    parts = tok * 3 * 128 * 2 + tok * 128 * 4 + tok * 4 + tok * 128 * 2 + 2 * 32 * 128 * 128 * 4
    total = 402_653_184 + 268_435_456 + 2_097_152 + 134_217_728 + 4_194_304
    assert parts == total == 811_597_824
    got = bench.prefill_bytes(2 * 8192, 2, 32, 128, 128, 2, state_in=False, per_key=True)
    assert got == 811_597_824


def test_prefill_bytes_varlen_workload():
    import gdn_synth as gs
    lengths = gs.generate(gs.small_case("varlen", decode_steps=0))["lengths"]
    tokens = sum(lengths)
    head_tokens = tokens * 16
    per_head_token = 3 * 128 * 2 + 128 * 2 + 4 + 4  # q, k, v, o, g, beta
    state = 64 * 16 * 128 * 128 * 4 * 2            # read and written
    assert per_head_token == 1032 and state == 134_217_728
    got = bench.prefill_bytes(tokens, 64, 16, 128, 128, 2, state_in=True, per_key=False)
    assert got == head_tokens * per_head_token + state


def test_backward_bytes_gdn_workload():
    # q, k, v, d_o read in bf16; g, beta read; dq, dk, dv, dg, dbeta written
    # in fp32; dstate_in written (the zero initial state is not read)
    tok = 4 * 4096 * 16
    parts = (tok * 4 * 128 * 2 + tok * 2 * 4 + tok * (128 + 128 + 128 + 1 + 1) * 4
             + 4 * 16 * 128 * 128 * 4)
    assert parts == 268_435_456 + 2_097_152 + 404_750_336 + 4_194_304 == 679_477_248
    assert bench.backward_bytes(4 * 4096, 4, 16, 128, 128, 2, False, False) == 679_477_248


def test_prefill_flops_per_head_token():
    C, d = 64, 128
    per_chunk = 3 * 2 * C * C * d + 2 * 2 * C * C * d + 3 * 2 * C * d * d
    assert per_chunk // C == 180_224
    assert bench.prefill_flops(C, 1, d, d) == 180_224 * C
    assert bench.prefill_flops(4 * 4096, 16, d, d) == 180_224 * 4 * 4096 * 16


def test_decode_bytes_per_update():
    assert bench.decode_bytes_per_update(128, 128, 2, False) == 2 * 65_536 + 768 + 256 + 8
    assert bench.decode_bytes_per_update(128, 128, 2, False) == 132_104
    # KDA: a gate per key channel
    assert bench.decode_bytes_per_update(128, 128, 2, True) == 132_104 + 127 * 4


def test_packed_decode_bytes_per_update():
    assert bench.decode_bytes_per_update_packed(128, 128, 2, False, "int8_g32") == 37_896
    assert (bench.decode_bytes_per_update_packed(128, 128, 2, False, "int8_g32")
            == 2 * 16_384 + 2 * 4 * 128 * 4 + 1_032)
    # FP8 tiles: one scale per 64 value columns
    assert (bench.decode_bytes_per_update_packed(128, 128, 2, False, "fp8_tile64")
            == 2 * 16_384 + 2 * 4 * 2 + 1_032)
    assert (bench.decode_bytes_per_update_packed(128, 128, 2, False, "int8_g16")
            == 2 * 16_384 + 2 * 4 * 128 * 8 + 1_032)


def test_recorded_traffic_only_for_its_sources(monkeypatch, tmp_path):
    import json
    import os
    prof = tmp_path / "profiles"
    prof.mkdir()
    h = bench.kernel_source_hash("decode")
    (prof / "traffic.json").write_text(json.dumps(
        {"decode": {"bytes_per_launch": 123, "source_hash": h},
         "backward": {"bytes_per_launch": 456, "source_hash": "0" * 16}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the sources are read from the package under ROOT: point it at the real one
    os.symlink(os.path.join(os.path.dirname(os.path.abspath(bench.__file__)),
                            "state_quantized_recurrence_b200"),
               tmp_path / "state_quantized_recurrence_b200")
    assert bench.recorded_traffic("decode") == 123
    assert bench.recorded_traffic("backward") is None        # taken on other sources
    assert bench.recorded_traffic("decode_packed") is None   # never recorded


def test_source_hash_follows_the_sources():
    # the two decode records are compiled from the same files
    assert bench.kernel_source_hash("decode") == bench.kernel_source_hash("decode_packed")
    assert bench.kernel_source_hash("decode") != bench.kernel_source_hash("backward")
    assert len(bench.kernel_source_hash("prefill_gdn")) == 16
