"""The benchmark's analytic step bound (bench.step_roofline) on the replay
workload: the mean bytes one decoder transition must move are the weights
(about 3.03 GB at bf16) plus the ring, the cross-attention memory reads and
the ring insert (about 37.1 GB averaged over t = 1..1023), which at the
measured copy bandwidth is about 6.1 ms per transition.  Also checks that the
bound scales with the work it counts, and that the reported DRAM traffic is
taken from an ncu summary only while the kernel source is the one captured."""
import bench
import synth

PEAKS = {"hbm_gbs": 6557.8, "bf16_tflops": 1663.7, "bf16_tflops_sustained": 1390.4, "source": "test"}


def test_replay_bound_per_transition():
    w = synth.workload("replay")
    r = bench.step_roofline(w, "replay", PEAKS)
    assert r["decoder_transitions"] == 1023
    d, L, F, V, B = w["d"], w["n_layers"], w["ffn"], w["vocab"], w["batch"]
    weights = 2 * (L * (6 * d * d + 3 * d * F) + 3 * d * d + V * d)
    assert abs(weights / 1e9 - 3.03) < 0.02
    kv = sum(B * 2 * 2 * d * (L * (min(t, 256) - 1) + L + L * t) for t in range(1, 1024)) / 1023
    assert abs(kv / 1e9 - 37.1) < 0.3
    enc_ms = (2 * B * 1024 * (L * (4 * d * d + 3 * d * F) + 2 * d * d) + 4 * B * L * d * 1024 * 1024 / 2) / 1390.4e12 * 1e3
    per_transition = (r["bound_ms"] - enc_ms) / 1023
    assert abs(per_transition - (weights + kv) / 6557.8e9 * 1e3) < 0.05
    assert 5.9 < per_transition < 6.4


def test_bound_grows_with_work():
    base = synth.workload("replay", prompt=256)
    b0 = bench.step_roofline(base, "replay", PEAKS)["bound_ms"]
    # twice the sequences: twice the KV bytes and FLOPs, the same weight bytes
    b2 = bench.step_roofline(dict(base, batch=512), "replay", PEAKS)["bound_ms"]
    assert 1.5 * b0 < b2 < 2 * b0
    # twice the tokens: twice the transitions, each reading a longer memory
    assert bench.step_roofline(dict(base, prompt=512), "replay", PEAKS)["bound_ms"] > 2 * b0
    g = synth.workload("small")
    assert bench.step_roofline(g, "generate", PEAKS)["decoder_transitions"] == g["prompt"] + g["gen"] - 1


def test_traffic_ratio_only_for_the_captured_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu summary only while the
    kernel source still has the SHA-1 recorded at capture time."""
    import hashlib

    import bench
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "stateful_decoder_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "attn_decode.cu").write_bytes(b"// kernel v1\n")
    sha = hashlib.sha1(b"// kernel v1\n").hexdigest()
    (tmp_path / "profiles" / "prefix_attn_replay.md").write_text(
        f"x\ntraffic_per_algorithmic_byte: 1.015\nkernel_source_sha1: {sha}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_traffic_ratio()[0] == 1.015
    (src / "attn_decode.cu").write_bytes(b"// kernel v2\n")
    ratio, note = bench.read_traffic_ratio()
    assert ratio is None and "changed" in note
