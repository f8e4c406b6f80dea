"""Host-side arithmetic of bench.py: the algorithmic bytes a decode reads,
the number of layers cycled to keep the cache out of L2, and the source hash
that ties a committed ncu summary to the kernel it measured.  CPU only."""

import bench
import workloads as W


def test_packed_kv_bytes_per_token_head():
    # 96 B per cached token-head (K and V codes 32 + 32, scale/zero 16 + 16),
    # 512 B per fp16 sink token-head (K and V rows of 128 halves)
    w = W.WORKLOADS["llama7b"]
    assert bench.packed_kv_bytes(w, w.seq_lens()) == 32 * 32768 * 96 == 100663296
    g = W.WORKLOADS["gqa_sinks"]
    assert bench.packed_kv_bytes(g, g.seq_lens()) == 8 * 8 * ((131072 - 4) * 96 + 4 * 512)
    t = W.custom(B=2, Hkv=3, sink=4)
    assert bench.packed_kv_bytes(t, [2, 10]) == 3 * (2 * 512) + 3 * (6 * 96 + 4 * 512)


def test_layers_keep_three_l2s_of_other_traffic_between_uses():
    L2 = bench.L2_BYTES
    assert bench.layers_for(3 * L2) == 1                 # one layer already exceeds it
    for size in (100663296, L2 // 2, L2 + 1):
        n = bench.layers_for(size)
        if n:
            assert (n - 1) * size >= 3 * L2 and (n - 2) * size < 3 * L2
    assert bench.layers_for(1 << 20) == 0                # too small: flush instead


def test_profile_traffic_is_tied_to_the_kernel_source(tmp_path, monkeypatch):
    sha = bench.kernel_source_sha()
    assert len(sha) == 16
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "decode_split_x.txt").write_text("source_sha256: %s\ndram_bytes_per_launch: 123\n" % sha)
    (prof / "decode_split_y.txt").write_text("source_sha256: 0000\ndram_bytes_per_launch: 123\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: sha)
    assert bench.profiled_traffic("x") == 123.0
    assert bench.profiled_traffic("y") is None           # taken on another kernel source
    assert bench.profiled_traffic("z") is None           # no summary
    # a summary taken on a smaller case scales to the full launch by the
    # ratio of algorithmic bytes (units processed)
    (prof / "decode_split_s.txt").write_text("source_sha256: %s\ndram_bytes_per_launch: 150\n"
                                             "algorithmic_bytes_per_launch: 100\n" % sha)
    assert bench.profiled_traffic("s", 400) == 600.0
    assert bench.profiled_traffic("s") == 150.0


def test_graph_plan_runs_exactly_the_requested_steps():
    for K in (1, 3, 20, 39, 40, 41, 100, 2000):
        for layers in (1, 5, 7):
            per, full, rem = bench.graph_plan(K, layers)
            assert per % layers == 0 and per >= layers
            assert per * full + rem == K and 0 <= rem < per


def test_oracle_sample_scale():
    # the median sequence of a ragged batch, and the factor from its
    # (sequence, heads) sample to the whole step's context token-heads
    assert bench.sample_sequence([5, 1, 9, 3]) == 3        # sorted 1, 3, 5, 9: lower middle
    assert bench.sample_sequence([7, 7, 7]) == 1
    w = W.WORKLOADS["ragged"]
    lens = w.seq_lens()
    b = bench.sample_sequence(lens)
    s = bench.sample_scale(w, lens, b, 2)
    assert abs(s * lens[b] * 2 - lens.sum() * 32) < 1e-6 * s
    u = W.WORKLOADS["llama7b"]
    assert bench.sample_scale(u, u.seq_lens(), 0, 4) == 32 / 4
