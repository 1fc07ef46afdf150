"""Host-side logic of the 52-layer denoise sweep (no GPU): the algorithmic
byte and weight counts the benchmark divides by, the per-layer seeds, and the
shape chain of the dense projections."""
import bench
import oracle
import synth


def test_sweep_packed_bytes_and_weights():
    wl = synth.WORKLOADS["denoise_sweep_52"]
    E, H, I = wl["num_experts"], wl["hidden"], wl["inter"]
    per_layer = 0
    for n, k, e in [(I, H, E), (H, I, E)] + [(n, k, 1) for n, k in wl["dense"]]:
        c, s = oracle.packed_bytes(n, k, e)
        per_layer += c + s
    assert bench.sweep_packed_bytes() == wl["layers"] * per_layer == 42_223_534_080
    # 5 bits per weight exactly
    assert bench.sweep_packed_bytes() * 8 == bench.sweep_weights() * 5
    assert bench.sweep_weights() == 67_557_654_528


def test_sweep_seeds_distinct():
    wl = synth.WORKLOADS["denoise_sweep_52"]
    seeds = [synth.sweep_seed(l, j) for l in range(wl["layers"]) for j in range(8)]
    assert len(set(seeds)) == len(seeds)
    # none collides with the seeds of the other workloads
    others = {v for name, d in synth.WORKLOADS.items() if name != "denoise_sweep_52"
              for key, v in d.items() if key.endswith("seed")}
    assert not others & set(seeds)


def test_sweep_dense_chain():
    wl = synth.WORKLOADS["denoise_sweep_52"]
    (n0, k0), (n1, k1) = wl["dense"]
    assert k0 == wl["hidden"] and n1 == wl["hidden"] and k1 == n0
    _, shapes = bench.sweep_shapes()
    assert [name for name, _ in shapes] == ["up", "down", "dense_in", "dense_out"]


def test_sweep_cpu_sample_runs():
    r = bench.sweep_cpu_sample(rows=2)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] == 1
