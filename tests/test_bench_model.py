"""The benchmark's analytic step bound (bench.step_roofline) on the replay
workload: the mean bytes one decoder transition must move are the weights
(about 3.03 GB at bf16) plus the ring, the cross-attention memory reads and
the ring insert (about 37.1 GB averaged over t = 1..1023), which at the
measured copy bandwidth is about 6.1 ms per transition.  The generation block
of the reference-depth model adds the encoder step's cache read.  Also checks
that the bound scales with the work it counts, that the metric string names
the model that ran, and that the reported DRAM traffic is taken from the ncu
record only while the kernel source is the one captured."""
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


def test_generation_block_bound():
    """One block of 32 generation transitions of the 48+48 model at B = 128:
    weights of the decoder transition and of the encoder step (10.8 GB),
    plus per position t the ring (255 entries once t > 256), the memory and
    encoder-cache reads of t positions and the inserts.  At t = 2400 that
    is about 256 GB, so about 39 ms per transition."""
    w = synth.workload("refdepth", block=32)
    d, L, F, V, B = w["d"], w["n_layers"], w["ffn"], w["vocab"], w["batch"]
    weights = 2 * (L * (6 * d * d + 3 * d * F) + 3 * d * d + V * d) + 2 * (L * (4 * d * d + 3 * d * F) + 2 * d * d)
    assert abs(weights / 1e9 - 10.8) < 0.1
    r = bench.step_roofline(w, "block", PEAKS, (2385, 2416))
    assert r["decoder_transitions"] == 32
    kv = sum(B * 4 * d * (L * 255 + L + L * t + L * t + L + 1) for t in range(2385, 2417))
    assert abs(r["bound_ms"] - (32 * weights + kv) / 6557.8e9 * 1e3) < 1e-6 * r["bound_ms"]
    assert 37 * 32 < r["bound_ms"] < 41 * 32
    # the mean over several blocks is per block
    r2 = bench.step_roofline(w, "block", PEAKS, (2385, 2448))
    assert r["bound_ms"] < r2["bound_ms"] < 1.05 * r["bound_ms"]


def test_metric_names_the_model_that_ran():
    assert bench.metric_name(synth.workload("refdepth"), "block") == \
        "RLT decoder tokens/s (B seqs, 48+48 tied) on 1 B200; % of step roofline"
    name = bench.metric_name(synth.workload("replay"), "replay")
    assert "24+24" in name and "48+48" not in name


def test_traffic_ratio_only_for_the_captured_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu record only while the
    kernel source still has the SHA-1 recorded at capture time."""
    import hashlib
    import json

    import bench
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "stateful_decoder_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "attn_decode.cu").write_bytes(b"// kernel v1\n")
    sha = hashlib.sha1(b"// kernel v1\n").hexdigest()
    rec = tmp_path / "profiles" / "traffic.json"
    rec.write_text(json.dumps({"prefix_attn": {"source": "stateful_decoder_b200/csrc/attn_decode.cu",
                                               "source_sha1": sha, "traffic_per_algorithmic_byte": 1.015,
                                               "case": "test"}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.read_traffic_ratio()[0] == 1.015
    (src / "attn_decode.cu").write_bytes(b"// kernel v2\n")
    ratio, note = bench.read_traffic_ratio()
    assert ratio is None and "changed" in note


def test_block_share_scale():
    """The prefix-attention share of the block step is measured on the two
    blocks after the timed ones and scaled by the ratio of mean attended keys
    (a launch at position t reads t keys)."""
    import bench
    scale, note = bench.block_share_scale((2209, 2848), 32, 2)
    prof = list(range(2852, 2913, 4))  # every 4th of t = 2849..2912
    assert abs(scale - 2528.5 / (sum(prof) / len(prof))) < 1e-12
    assert "t=2852..2912" in note and "t=2209..2848" in note
